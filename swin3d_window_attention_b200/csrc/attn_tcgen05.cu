// Shifted-window attention on the sm_100a tensor cores (tcgen05.mma, accumulators in
// TMEM), one persistent CTA per SM, warp-specialised.
//
// Method: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models".
//  * section "CuTe DSL window attention": per (window, head) S = scale * Q K^T, the Swin
//    shift mask, row softmax in FP32, O = softmax(S) V with the whole window's K and V
//    resident in shared memory (N = 144 <= tile, the single-stage case), nothing N x N in
//    global memory; BF16 operands with FP32 softmax (BF16_MIXED);
//  * section "Kernel fusion for backbone memory traffic": the cyclic shift, padding and
//    3D window partition, and the inverse merge / un-shift, are folded into the gather of
//    Q/K/V rows straight from grid layout and the scatter of O rows straight back to grid
//    layout, so none of them costs a global-memory pass.
//
// Work unit ("tile"): one (sample, window, head).  Roles (warp -> SM sub-partition w % 4):
//   softmax warps 0-7  warp w owns TMEM lanes 32 (w % 4) .. +31 = query rows of
//                      S0 = Q[0:128] K^T, and of each row the keys of half w / 4 (key
//                      groups 2k + h of 8 keys, 72 keys).  It reads its 72 logits out of
//                      TMEM once (releasing S for the next tile), takes the masked max, swaps
//                      it with the warp holding the other half, then exp2 and P rounded to
//                      bf16 into shared memory.  One tile later (the PV MMA overlaps the next
//                      softmax) it loads half of the row's O columns and the row sum (an MMA
//                      output column, see below), scales by 1/rowsum, rounds to nearest even
//                      and stores them to the query's original grid position in 32-byte
//                      pieces, lane pairs swapping one so that each store writes both of a
//                      row's pieces; padded slots are dropped.
//   tail warp 8        the same for the 16 tail rows (S1 = Q[128:144] K^T in TMEM lanes
//                      0..15, reachable from warp 8 like from warp 0), read with the 16x32bx2
//                      shape: threads 0..15 hold half 0 of rows 128..143, threads 16..31
//                      half 1; the two halves swap row maxima by a shuffle.
//   MMA warp 9         the warp runs the issue loop, lane 0 issues: S(t+1) as soon as tile
//                      t+1 is loaded and S(t) has left TMEM, then PV(t) = P V once P(t) is in
//                      shared memory (main rows and tail rows handed over separately), with V
//                      read as an MN-major operand followed by 16 columns of ones, so O's
//                      columns from 64 on are the row sums of the bf16 P; completion is
//                      signalled by tcgen05.commit.
//   TMA warp 10        (attn_common.cuh, shared with the TF32 kernel)
//                      one thread loads the tile's Q, K and V with TMA, a T-slab (win_h x
//                      win_w tokens) at a time: one box per slab, or with a W shift two
//                      (the w offsets before the wrap-around split, then the rest, which is
//                      also the slots' order), each cut in two at the H seam; straight from
//                      grid layout into a 3-stage ring in the tensor core's 128-byte swizzled
//                      K-major layout; padded coordinates are out of bounds and read as zero.
//                      It runs ahead as far as the ring allows.
//   table warp 11      (attn_common.cuh) writes the slot -> grid-token table, a bitmask of the real slots, the
//                      window's "last along a shifted axis" flags and, from these, the key
//                      masks per region combination and key half, for the stage being loaded.
// Synchronisation is by mbarriers only; every wait is bounded by a time limit and a
// timeout unwinds the whole CTA (error word set, copies drained, TMEM freed).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"
#include "s3w_internal.h"
#include "sm100_ptx.cuh"

namespace s3w {
namespace {

using namespace sm100;
using namespace attn;

// Stages of the Q/K/V ring: three for the attention kernel (two are 60% slower); two in the
// fused kernel, where three measure the same because its AdaLN warps set the pace.
constexpr int kStagesPlain = 3;
constexpr int kStagesFused = 2;
constexpr int kTileBytes = kChunkTileBytes;         // 18432: one of Q / K / V
constexpr int kStageBytes = 3 * kTileBytes;         // 55296

// Shared-memory map (offsets from a 1024-byte aligned base).  The tail P blocks only hold
// 16 rows; the rows 16..127 their M = 128 descriptors also cover fall on the buffers that
// follow (valid memory, results of those rows are never used).
constexpr int OFF_P1B0 = 0;        // tail P rows 0..15, keys 0..63   (128B swizzle)
constexpr int OFF_P1B1 = 2048;     // tail P rows 0..15, keys 64..127 (128B swizzle)
constexpr int OFF_P1B2 = 4096;     // tail P rows 0..15, keys 128..143 (32B swizzle)
constexpr int OFF_P0B0 = 5120;     // P rows 0..127, keys 0..63
constexpr int OFF_P0B1 = OFF_P0B0 + 16384;
constexpr int OFF_P0B2 = OFF_P0B1 + 16384;   // keys 128..143, 32B swizzle, 4 KB
constexpr int OFF_STAGE = OFF_P0B2 + 4096;   // 41984 (1024-aligned)
constexpr int kOnesBytes = 16 * kRowBytes;
constexpr int kXchgFloats = 2 * 2 * 128;

template <bool FUSED>
struct SmemLayout {
  static constexpr int kStages = FUSED ? kStagesFused : kStagesPlain;
  // 16 key rows of bf16 ones in the V operand's layout: the PV MMA reads them as 16 more
  // output columns (through the descriptor's leading byte offset), so every such column of
  // O is the row sum of P as rounded to bf16, the exact normaliser of the P the MMA used.
  static constexpr int OFF_ONES = OFF_STAGE + kStages * kStageBytes;
  static constexpr int OFF_TABLE = OFF_ONES + kOnesBytes;
  static constexpr int OFF_SLOTC = OFF_TABLE + kStages * kTableBytes;
  static constexpr int OFF_BARS = OFF_SLOTC + kSlotConstBytes;
  // barriers: load[S] (TMA bytes), empty[S], table[S], s_full, s_empty, p_full, p_empty,
  // o_full, o_empty, drain, row max written[0][2], tail p_full, tail p_empty, row max
  // written[1][2] (row max barriers: [tile parity][key half]).  A softmax thread releases S
  // (s_empty) before it waits for the other half's row maximum, so the warps of one half
  // can reach tile t+2 before a warp of the other half has waited for tile t; one row-max
  // barrier per tile parity keeps that wait on its own phase.
  static constexpr int kNumBars = 3 * kStages + 13;
  // Row max of each key half of the main rows, exchanged between the two warps that share
  // a row: [tile parity][key half][row].
  static constexpr int OFF_XCHG = OFF_BARS + kNumBars * 8;
  static constexpr int OFF_MISC = OFF_XCHG + kXchgFloats * 4;   // tmem address, abort flag, producer stop
  static constexpr int kPlainBytes = OFF_MISC + 16;
  // Fused attention + AdaLN only: per window parity, the running statistics of every row's
  // two column halves, the rows' grid tokens, and the window-ready / window-free barriers.
  static constexpr int OFF_WSTAT = kPlainBytes;                  // float2 [2 parity][2 half][kN]
  static constexpr int OFF_WTOK = OFF_WSTAT + 2 * 2 * kN * 8;     // int [2 parity][kN]
  static constexpr int OFF_WBAR = OFF_WTOK + 2 * kN * 4;          // win_full[2], win_free[2]
  static constexpr int kBytes = FUSED ? OFF_WBAR + 4 * 8 : kPlainBytes;
  static constexpr int kAlloc = kBytes + 1024;                    // slack for the 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// TMEM columns (fp32 accumulators, lane = row).  Every MMA destination is 32-aligned.  O
// has 80 columns: the head's outputs (the first head_dim of 64), then from column 64 on 16
// copies of the row sum.
constexpr uint32_t TM_S0 = 0, TM_S1 = 160, TM_O0 = 320, TM_O1 = 416;
constexpr uint32_t kOnesCol = 64;
constexpr uint32_t kTmemCols = 512;

constexpr int kThreads = 384;
constexpr int kMainWarps = 8;          // rows 0..127: warp w holds lanes 32 (w % 4) .., keys 72 (w / 4) ..
constexpr int kTailWarp = 8;           // tail rows 128..143 (TMEM lane quarter 0, like warp 0)
constexpr int kMmaWarp = 9;
constexpr int kTmaWarp = 10;
constexpr int kFirstProducerWarp = 11;
constexpr int kProducerThreads = 32;   // table writer (warp 11)
// Fused attention + AdaLN: warps 12..15 normalise finished windows (the AdaLN warps).
constexpr int kThreadsFused = 512;
constexpr int kFirstAdalnWarp = 12;
constexpr int kAdalnThreads = 128;

// Operand descriptors.  K-major 128B swizzle: 8-row x 128-byte atoms, 1024 bytes apart.
// K-major 32B swizzle: 8-row x 32-byte atoms, 256 bytes apart.  MN-major 128B swizzle (V,
// whose rows are keys = the K dimension): 8-key x 64-element atoms, 1024 bytes apart along
// K; the leading byte offset is the distance to the next 64 elements along N.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128B); }
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t addr) { return smem_desc(addr, 16, 256, kSwizzle32B); }

// ---------------------------------------------------------------- fused attention + AdaLN
// "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models", section
// "Kernel fusion for backbone memory traffic": LayerNorm, FiLM modulation and the residual
// add fused without a full-width intermediate.  The fused kernel takes whole windows (all
// heads of every token of the window pass through one CTA).  Per head, the epilogue rounds
// the thread's half-row of O to bf16 (the AdaLN input, exactly what the unfused path stores),
// merges its statistics into a running (mean, M2) per (row, column half) (Chan, Golub and
// LeVeque's pairwise update), and writes the bf16 values to the CTA's workspace.  When the
// last head is in, the AdaLN warps normalise the window row by row:
//   out = residual + (x - mean) / sqrt(var + eps) * (1 + scale_b) + shift_b.

// Epilogue of one (window, head) tile in the fused kernel: the thread holds HD / 2 values of
// O (its column half: groups of 16 at 32m + 16 half) already summed over the keys.
template <int HD>
__device__ __forceinline__ void fused_epilogue(const WinGeom& g, const AdalnArgs& fa, void* o, const float* ov,
                                               float inv, int head, int tok, int row, int half, int wp,
                                               float2* wstat, int* wtok, int C) {
  constexpr int kVals = HD / 2;
  uint32_t u[kVals / 2];
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < kVals / 2; ++e) {
    u[e] = pack_bf16x2(ov[2 * e] * inv, ov[2 * e + 1] * inv);
    sum += __uint_as_float(u[e] << 16) + __uint_as_float(u[e] & 0xffff0000u);
  }
  const float mean_b = sum * (1.0f / kVals);
  float m2_b = 0.f;
#pragma unroll
  for (int e = 0; e < kVals / 2; ++e) {
    const float d0 = __uint_as_float(u[e] << 16) - mean_b, d1 = __uint_as_float(u[e] & 0xffff0000u) - mean_b;
    m2_b = fmaf(d0, d0, fmaf(d1, d1, m2_b));
  }
  float2& st = wstat[(wp * 2 + half) * kN + row];
  if (head == 0) {
    st = make_float2(mean_b, m2_b);
    if (half == 0) wtok[wp * kN + row] = tok;
  } else {
    // merge n_a = head * kVals values (mean_a, M2_a) with n_b = kVals values (mean_b, M2_b)
    const float2 a = st;
    const float na = static_cast<float>(head * kVals), nb = static_cast<float>(kVals);
    const float n = na + nb, d = mean_b - a.x;
    st = make_float2(a.x + d * (nb / n), a.y + m2_b + d * d * (na * nb / n));
  }
  if (tok < 0) return;
  uint16_t* ws = fa.ws + ((static_cast<long long>(blockIdx.x) * 2 + wp) * kN + row) * C + head * HD;
#pragma unroll
  for (int m = 0; m < HD / 32; ++m) {
    const int col = 32 * m + 16 * half;
    uint32_t v8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v8[e] = u[8 * m + e];
    st_global_v8(ws + col, v8);
    if (o != nullptr)
      st_global_v8(static_cast<uint16_t*>(o) + static_cast<long long>(tok) * g.o_stride + head * HD + col, v8);
  }
}

// The AdaLN warps (warps 12..15): per finished window, warp q normalises rows q, q + 4, ...,
// two rows per pass; lane l owns the 16-channel blocks l, l + 32, ... of each row.  A block
// moves with one 32-byte load of x (bf16, from the workspace), two of the residual and one
// or two 32-byte stores, and the per-channel factors 1 + scale and shift of a lane's block
// stay in registers for the whole window when each lane has at most one block (C <= 512):
// the warps' global loads and stores share the SM's memory-instruction queue with the
// softmax warps' shared- and tensor-memory traffic, so the fewer of them the better.  Every
// load of a pass is issued before its first store (the output may be the residual itself,
// so the compiler could not reorder them).  The two column halves' running statistics of a
// row combine into the row's mean and variance (biased, over C); then, per element,
//   y = x * g + (r + shift - mean * g),   g = rstd * (1 + scale),
// in packed two-lane fp32 arithmetic.
// wbar0: the window barriers, win_full[2] then win_free[2].
struct AdalnBlockIn {
  uint32_t x[8];    // 16 bf16 of x
  uint32_t r[16];   // 16 fp32 of the residual (bit patterns)
};

__device__ __forceinline__ void adaln_block_load(const uint16_t* xrow, const float* rrow, int cb, AdalnBlockIn& in) {
  ld_global_v8(xrow + cb * 16, in.x);
  uint32_t (&r0)[8] = *reinterpret_cast<uint32_t(*)[8]>(&in.r[0]);
  uint32_t (&r1)[8] = *reinterpret_cast<uint32_t(*)[8]>(&in.r[8]);
  ld_global_cs_v8(rrow + cb * 16, r0);
  ld_global_cs_v8(rrow + cb * 16 + 8, r1);
}

__device__ __forceinline__ void adaln_block_store(const AdalnArgs& fa, int tok, int cb, int C, float mean, float rstd,
                                                  const AdalnBlockIn& in, const float (&sc1)[16],
                                                  const float (&sh)[16]) {
  const float2 rs = make_float2(rstd, rstd), nm = make_float2(-mean, -mean);
  float y[16];
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const uint32_t u = in.x[e >> 1];
    const float2 x = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    const float2 gg = mul2(rs, make_float2(sc1[e], sc1[e + 1]));
    const float2 bb = fma2(nm, gg, make_float2(sh[e], sh[e + 1]));
    const float2 t = add2(make_float2(__uint_as_float(in.r[e]), __uint_as_float(in.r[e + 1])), bb);
    const float2 yy = fma2(x, gg, t);
    y[e] = yy.x;
    y[e + 1] = yy.y;
  }
  if (fa.out_f32) {
    float* op = static_cast<float*>(fa.out) + static_cast<long long>(tok) * C + cb * 16;
    uint32_t v0[8], v1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v0[e] = __float_as_uint(y[e]);
      v1[e] = __float_as_uint(y[8 + e]);
    }
    st_global_cs_v8(op, v0);
    st_global_cs_v8(op + 8, v1);
  } else {
    uint32_t v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
    st_global_cs_v8(static_cast<__nv_bfloat16*>(fa.out) + static_cast<long long>(tok) * C + cb * 16, v);
  }
}

__device__ __forceinline__ void adaln_factors(const float* scb, const float* shb, int cb, float (&sc1)[16],
                                              float (&sh)[16]) {
  uint32_t a[8], b[8];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    ld_global_v8(scb + cb * 16 + 8 * h, a);
    ld_global_v8(shb + cb * 16 + 8 * h, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sc1[8 * h + e] = 1.0f + __uint_as_float(a[e]);
      sh[8 * h + e] = __uint_as_float(b[e]);
    }
  }
}

__device__ __forceinline__ void adaln_warps(const WinGeom& g, const AdalnArgs& fa, const float2* wstat,
                                            const int* wtok, uint32_t wbar0, volatile int* abort_flag, int* err,
                                            unsigned long long limit_ns, int warp, int lane, int C) {
  auto win_full = [&](int wp) { return wbar0 + 8u * wp; };
  auto win_free = [&](int wp) { return wbar0 + 8u * (2 + wp); };
  const int q = warp - kFirstAdalnWarp;
  const float nh = 0.5f * static_cast<float>(C);   // values per column half of a row
  const int nb = C >> 4;                            // 16-channel blocks per row
  const bool hoisted = nb <= 32;                    // at most one block per lane
  bool aborted = false;
  for (int k = 0;; ++k) {
    const long long win = blockIdx.x + static_cast<long long>(k) * gridDim.x;
    if (win >= g.windows) break;
    const int wp = k & 1;
    if (__any_sync(0xffffffffu, *abort_flag != 0)) {
      aborted = true;
      break;
    }
    const long long b = fdiv(static_cast<int>(win), g.div_per_sample);
    const float* scb = fa.scale + b * C;
    const float* shb = fa.shift + b * C;
    float sc1[16], sh[16];
    if (hoisted && lane < nb) adaln_factors(scb, shb, lane, sc1, sh);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(win_full(wp), (k >> 1) & 1, limit_ns))) {
      aborted = true;
      break;
    }
    const uint16_t* wsw = fa.ws + (static_cast<long long>(blockIdx.x) * 2 + wp) * kN * C;
    const int* tokw = wtok + wp * kN;
    // this warp's rows: j-th row q + 4j; rows at or beyond the window size are padding
    // slots (rows 128.. exist only with a tail warp)
    const int nrows = g.N > q ? (g.N - q + 3) / 4 : 0;
    auto stats = [&](int r, float& mean, float& rstd) {
      const float2 s0 = wstat[(wp * 2 + 0) * kN + r], s1 = wstat[(wp * 2 + 1) * kN + r];
      const float d = s1.x - s0.x;
      mean = 0.5f * (s0.x + s1.x);
      const float var = (s0.y + s1.y + d * d * (0.5f * nh)) / static_cast<float>(C);
      rstd = 1.0f / sqrtf(var + fa.eps);
    };
    for (int j = 0; j < nrows; j += 2) {
      const int ra = q + 4 * j, rb = ra + 4;
      const int ta = tokw[ra];
      const int tb = j + 1 < nrows ? tokw[rb] : -1;
      float ma = 0.f, sa = 0.f, mb = 0.f, sb = 0.f;
      if (ta >= 0) stats(ra, ma, sa);
      if (tb >= 0) stats(rb, mb, sb);
      const float* resa = fa.residual + static_cast<long long>(ta >= 0 ? ta : 0) * C;
      const float* resb = fa.residual + static_cast<long long>(tb >= 0 ? tb : 0) * C;
      const uint16_t* xa = wsw + static_cast<long long>(ra) * C;
      const uint16_t* xb = wsw + static_cast<long long>(rb) * C;
#pragma unroll 1
      for (int cb = lane; cb < nb; cb += 32) {
        AdalnBlockIn ina, inb;
        if (ta >= 0) adaln_block_load(xa, resa, cb, ina);
        if (tb >= 0) adaln_block_load(xb, resb, cb, inb);
        if (!hoisted) adaln_factors(scb, shb, cb, sc1, sh);
        if (ta >= 0) adaln_block_store(fa, ta, cb, C, ma, sa, ina, sc1, sh);
        if (tb >= 0) adaln_block_store(fa, tb, cb, C, mb, sb, inb, sc1, sh);
      }
    }
    __syncwarp();
    mbar_arrive(win_free(wp));   // this thread has read the window's buffers of this parity
  }
  if (aborted) {
    if (lane == 0) record_error(err, kStatusTimeout);
    *abort_flag = 1;
  }
}

template <int HD, bool OUT_F32, bool FUSED>
__global__ void __launch_bounds__(FUSED ? kThreadsFused : kThreads, 1)
window_attn_tc_kernel(const __grid_constant__ WinGeom g, const __grid_constant__ TmaMaps maps,
                      void* __restrict__ o, int* __restrict__ err, unsigned long long limit_ns,
                      const __grid_constant__ AdalnArgs fa) {
  using L = SmemLayout<FUSED>;
  constexpr int kStages = L::kStages;
  constexpr int OFF_ONES = L::OFF_ONES, OFF_TABLE = L::OFF_TABLE, OFF_SLOTC = L::OFF_SLOTC, OFF_BARS = L::OFF_BARS;
  constexpr int OFF_XCHG = L::OFF_XCHG, OFF_MISC = L::OFF_MISC;
  constexpr int OFF_WSTAT = L::OFF_WSTAT, OFF_WTOK = L::OFF_WTOK, OFF_WBAR = L::OFF_WBAR;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  Table* tables = reinterpret_cast<Table*>(sm + OFF_TABLE);
  const uint32_t bar0 = sb + OFF_BARS;
  auto load_bar = [&](int s) { return bar0 + 8u * s; };                  // Q/K/V of the stage landed
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };      // stage free again
  auto table_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };  // the stage's table written
  const uint32_t s_full = bar0 + 8u * (3 * kStages + 0);
  const uint32_t s_empty = bar0 + 8u * (3 * kStages + 1);
  const uint32_t p_full = bar0 + 8u * (3 * kStages + 2);
  const uint32_t p_empty = bar0 + 8u * (3 * kStages + 3);
  const uint32_t o_full = bar0 + 8u * (3 * kStages + 4);
  const uint32_t o_empty = bar0 + 8u * (3 * kStages + 5);
  const uint32_t drain_bar = bar0 + 8u * (3 * kStages + 6);
  // key half h of a tile of parity par wrote its row maxima
  auto xmax_bar = [&](int par, int h) { return bar0 + 8u * (3 * kStages + (par ? 11 : 7) + h); };
  // P of the main rows and of the tail rows are handed over separately, so the main rows'
  // next P may be written as soon as their own PV MMAs have read it.
  const uint32_t p_full_t = bar0 + 8u * (3 * kStages + 9);
  const uint32_t p_empty_t = bar0 + 8u * (3 * kStages + 10);
  float* xmax = reinterpret_cast<float*>(sm + OFF_XCHG);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* prod_stop = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);
  float2* wstat = reinterpret_cast<float2*>(sm + OFF_WSTAT);
  int* wtok = reinterpret_cast<int*>(sm + OFF_WTOK);
  auto win_full = [&](int wp) { return sb + OFF_WBAR + 8u * wp; };        // window's x and statistics written
  auto win_free = [&](int wp) { return sb + OFF_WBAR + 8u * (2 + wp); };  // window normalised: buffers free
  const int C = g.heads * HD;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long num_tiles = g.windows * g.heads;
  const bool has_tail = g.N > 128;
  const uint32_t n_soft = has_tail ? 288u : 256u;   // softmax threads: main rows (+ tail warp)

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(load_bar(s), 1);                        // the TMA thread's expect_tx arrival + bytes
      mbar_init(empty_bar(s), 1 + n_soft);              // PV commit + every softmax thread (table read)
      mbar_init(table_bar(s), kProducerThreads);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, n_soft);
    mbar_init(p_full, 256);
    mbar_init(p_empty, 1);
    mbar_init(p_full_t, 32);
    mbar_init(p_empty_t, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, n_soft);
    mbar_init(drain_bar, 1);
    for (int par = 0; par < 2; ++par)
      for (int h = 0; h < 2; ++h) mbar_init(xmax_bar(par, h), 128);
    if constexpr (FUSED) {
      for (int wp = 0; wp < 2; ++wp) {
        mbar_init(win_full(wp), n_soft);
        mbar_init(win_free(wp), kAdalnThreads);
      }
    }
    *abort_flag = 0;
    *prod_stop = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  SlotConst* slotc = reinterpret_cast<SlotConst*>(sm + OFF_SLOTC);
  init_slot_consts(g, slotc, tid);
  constexpr int kNT = FUSED ? kThreadsFused : kThreads;
  for (int i = tid; i < kOnesBytes / 16; i += kNT)   // bf16 1.0 = 0x3f80
    *reinterpret_cast<uint4*>(sm + OFF_ONES + 16 * i) = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  fence_proxy_async_smem();
  // Slots N..143 are never loaded: keep them zero (finite) for the whole kernel.
  if (g.N < kN) {
    for (int i = tid; i < kStages * 3 * (kN - g.N) * (kRowBytes / 16); i += kNT) {
      const int chunk = i % (kRowBytes / 16);
      const int rest = i / (kRowBytes / 16);
      const int r = g.N + rest % (kN - g.N);
      const int tile_id = rest / (kN - g.N);   // stage * 3 + tensor
      *reinterpret_cast<uint4*>(sm + OFF_STAGE + tile_id * kTileBytes + r * kRowBytes + chunk * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sb + OFF_MISC, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const Ring ring{sb + OFF_STAGE, load_bar(0), empty_bar(0), table_bar(0)};
  if (warp == kTmaWarp) {
    if (lane == 0)
      tma_loader<1, 64, kStages, kStageBytes, FUSED>(g, maps, ring, HD, num_tiles, abort_flag, err, limit_ns);
  } else if (warp == kFirstProducerWarp) {
    table_writer<kStages, FUSED>(g, tables, slotc, ring, num_tiles, abort_flag, prod_stop, err, limit_ns, lane);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // Issue order: S(t+1) goes out as soon as tile t+1 is loaded and S(t) has been read
    // out of TMEM, before PV(t); the softmax warps then find S(t+1) ready when they finish
    // tile t, and PV(t) runs underneath the softmax of tile t+1.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, kN, false, false);
    // N = 64 V columns (the box is 64 channels wide for head_dim 32 too) + 16 ones columns
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, kOnesCol + 16, false, true);
    static_assert(kN / 16 == 9, "the PV chain covers 144 keys");
    // Operand descriptors are linear in the address field (bits 0..13 = address / 16, every
    // operand below 256 KB), so each MMA's descriptor is a base plus a constant: the stage
    // moves it by kStageBytes / 16, a K step by 32 B (K-major) or 16 keys = 2048 B (V).
    const uint64_t dq0 = desc_kmajor_sw128(sb + OFF_STAGE);                    // Q of stage 0
    // V of stage 0; its second 64-column atom along N (leading byte offset) is the ones block
    const uint64_t dv0 = smem_desc(sb + OFF_STAGE + 2 * kTileBytes, OFF_ONES - (OFF_STAGE + 2 * kTileBytes), 1024,
                                   kSwizzle128B);
    const uint64_t dp0 = desc_kmajor_sw128(sb + OFF_P0B0), dp0b = desc_kmajor_sw32(sb + OFF_P0B2);
    const uint64_t dp1 = desc_kmajor_sw128(sb + OFF_P1B0), dp1b = desc_kmajor_sw32(sb + OFF_P1B2);
    constexpr uint64_t kStageStep = kStageBytes >> 4;
    const uint32_t leader = lane == 0 ? 1u : 0u;
    bool issued = false;
    auto issue_s = [&](int jt) -> bool {   // S(jt) = Q K^T of the tile in stage jt % kStages
      const int s = jt % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(load_bar(s), (jt / kStages) & 1, limit_ns))) return false;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_empty, (jt & 1) ^ 1, limit_ns))) return false;
      fence_proxy_async_smem();
      tc_fence_after();
      const uint64_t qd = dq0 + s * kStageStep, kd = qd + (kTileBytes >> 4);
      umma_chain_qk<HD / 16>(tmem + TM_S0, qd, kd, idesc_s, leader);
      if (has_tail) umma_chain_qk<HD / 16>(tmem + TM_S1, qd + ((128 * kRowBytes) >> 4), kd, idesc_s, leader);
      umma_commit_leader(s_full, leader);
      issued = true;
      return true;
    };
    auto issue_pv = [&](int jt) -> bool {  // O(jt) = P V of the tile in stage jt % kStages
      const int s = jt % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full, jt & 1, limit_ns))) return false;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_empty, (jt & 1) ^ 1, limit_ns))) return false;
      tc_fence_after();
      // Moving V by d (bytes / 16) moves the ones block's leading offset by -d.
      const uint64_t dstage = s * kStageStep;
      const uint64_t vd = dv0 + dstage - (dstage << 16);
      umma_chain_pv(tmem + TM_O0, dp0, vd, idesc_o, leader, dp0b, ((OFF_P0B1 - OFF_P0B0) >> 4) - 6);
      umma_commit_leader(p_empty, leader);
      if (has_tail) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full_t, jt & 1, limit_ns))) return false;
        tc_fence_after();
        umma_chain_pv(tmem + TM_O1, dp1, vd, idesc_o, leader, dp1b, ((OFF_P1B1 - OFF_P1B0) >> 4) - 6);
      }
      if (has_tail) umma_commit_leader(p_empty_t, leader);
      umma_commit_leader(o_full, leader);
      umma_commit_leader(empty_bar(s), leader);
      return true;
    };
    // Step j issues S(j) (if tile j exists) and then PV(j-1): S(0); S(1), PV(0); S(2), PV(1); ...
    // The whole warp runs this (every wait's outcome is agreed by a vote); lane 0 alone
    // issues the MMAs and commits.
    // Failure injection (tests): wait on the drain barrier, which nothing signals before the
    // loop below has run, so the bounded wait expires and the CTA takes the timeout path.
    bool ok = !g.test_stall || __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, limit_ns));
    const long long my_units = FUSED ? g.windows : num_tiles;   // windows (fused) or tiles
    const long long my_tiles =
        (static_cast<long long>(blockIdx.x) < my_units ? (my_units - 1 - blockIdx.x) / gridDim.x + 1 : 0) *
        (FUSED ? g.heads : 1);
    for (long long j = 0; ok && j <= my_tiles; ++j) {
      ok = !__any_sync(0xffffffffu, *abort_flag != 0);
      if (ok && j < my_tiles) ok = issue_s(static_cast<int>(j));
      if (ok && j > 0) ok = issue_pv(static_cast<int>(j - 1));
    }
    if (!ok && lane == 0) {
      record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
    // Drain: wait (bounded, independent of the test limit) until every MMA issued has
    // completed, so TMEM can be released.
    if (lane == 0 && issued) {
      umma_commit(drain_bar);
      if (!mbar_wait_bounded(drain_bar, 0, 2000000000ull)) record_error(err, kStatusTimeout);
    }
    __syncwarp();
  } else if (FUSED && warp >= kFirstAdalnWarp) {
    if constexpr (FUSED) adaln_warps(g, fa, wstat, wtok, sb + OFF_WBAR, abort_flag, err, limit_ns, warp, lane, C);
  } else if (warp < kMainWarps || (warp == kTailWarp && has_tail)) {
    // ------------------------------------------------------------------ softmax + epilogue
    // Every softmax thread owns one (query row, key half) and runs the same code.  Half h
    // holds the key groups 2k + h (k = 0..8) of 8 keys each, 72 keys.  Main warp w: row
    // 32 (w % 4) + lane (its TMEM lane in S0 = Q[0:128] K^T), half w / 4, read with the
    // 32x32b shape at column 16k + 8h; its partner (same row, other half) is warp w ^ 4,
    // and the two swap row max and row sum through shared memory.  Tail warp 8: row
    // 128 + lane % 16 (TMEM lane lane % 16 of S1 = Q[128:144] K^T), half lane / 16, read
    // with the 16x32bx2 shape (threads 16..31 see the columns 8 further on); its partner is
    // lane ^ 16 of the same warp (a shuffle).
    const bool is_tail = warp == kTailWarp;
    const float c = g.scale_log2;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int half = is_tail ? (lane >> 4) : ((warp >> 2) & 1);
    const int row = is_tail ? 128 + (lane & 15) : (warp & 3) * 32 + lane;
    const int lrow = is_tail ? (lane & 15) : row;   // row inside its P blocks
    const uint32_t pb0 = sb + (is_tail ? OFF_P1B0 : OFF_P0B0);
    const uint32_t pb1 = sb + (is_tail ? OFF_P1B1 : OFF_P0B1);
    const uint32_t pb2 = sb + (is_tail ? OFF_P1B2 : OFF_P0B2);
    const uint32_t s_base = is_tail ? tmem + TM_S1 : tmem + lane_base + TM_S0 + 8 * half;
    // O columns of a thread: groups of 16, 32m + 16h .. +15 (m < head_dim / 32); the main
    // rows take them with 32x32b at that column, the tail with 16x32bx2 at column 32m.
    const uint32_t o_base = is_tail ? tmem + TM_O1 : tmem + lane_base + TM_O0 + 16 * half;
    const uint32_t my_hi = [&] {
      uint32_t h = 0;
#pragma unroll
      for (int a = 0; a < 3; ++a) h |= ((slotc->hi[a][row >> 5] >> (row & 31)) & 1u) << a;
      return h;
    }();
    int it = 0;
    // state of the previous tile, finished one iteration later
    bool have_prev = false;
    int prev_it = 0, prev_head = 0, prev_tok = -1;
    bool aborted = false;


    // Epilogue of a finished tile: this thread's O columns and the row sum (column 64 of O)
    // from TMEM, scaled by 1/rowsum, stored to the grid position of the query slot
    // (padded slots dropped).
    auto epilogue = [&](int pit, int head, int tok) -> bool {
      const int k = fdiv(pit, g.div_heads);   // the CTA's window index (fused order)
      const int wp = k & 1;
      if constexpr (FUSED) {
        // the window's buffers of this parity must have been normalised (window k - 2)
        if (head == 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(win_free(wp), ((k >> 1) & 1) ^ 1, limit_ns)))
          return false;
      }
      bool ok = mbar_wait_bounded(o_full, pit & 1, limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      tc_fence_after();
      float ov[HD / 2];
      float l;
      if (!is_tail) {
#pragma unroll
        for (int m = 0; m < HD / 32; ++m) tmem_ld16(o_base + 32 * m, ov + 16 * m);
        tmem_ld1(o_base - 16 * half + kOnesCol, &l);
      } else {
#pragma unroll
        for (int m = 0; m < HD / 32; ++m) tmem_ld_16x32bx2_x16(o_base + 32 * m, ov + 16 * m);
        tmem_ld_16x32bx2_x1(o_base + kOnesCol, &l);
      }
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < HD / 32; ++m) reg_fence16(ov + 16 * m);
      reg_fence1(&l);
      tc_fence_before();
      mbar_arrive(o_empty);
      const float inv = l > 0.f ? rcp_approx(l) : 0.f;
      if constexpr (FUSED) {
        fused_epilogue<HD>(g, fa, o, ov, inv, head, tok, row, half, wp, wstat, wtok, C);
        if (head == g.heads - 1) {
          __threadfence_block();
          mbar_arrive(win_full(wp));   // this thread's share of the window is written
        }
        return true;
      }
      store_o_row<HD, OUT_F32>(o, g.o_stride, g.o_rows_32b != 0, tok, head, half, lane, ov, inv);
      return true;
    };

    // The thread's 72 logits are read from TMEM once (nine 8-column loads) and stay in
    // registers.  If any thread of the warp has a masked key (near the shift seams and the
    // padding), masked keys become -inf first, hence weight 0.
    auto selb = [](uint32_t w, int e, float x) { return ((w >> e) & 1u) ? x : -INFINITY; };
    auto row_max = [&](float (&x)[72], const uint4 mq) -> float {
      if (!is_tail) {
#pragma unroll
        for (int k = 0; k < 9; ++k) tmem_ld8(s_base + 16 * k, x + 8 * k);
      } else {
#pragma unroll
        for (int k = 0; k < 9; ++k) tmem_ld_16x32bx2_x8(s_base + 16 * k, x + 8 * k);
      }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 9; ++k) reg_fence8(x + 8 * k);
      if (__any_sync(0xffffffffu, mq.w != 0u)) {
#pragma unroll
        for (int k = 0; k < 9; ++k) {
          const uint32_t kb = k < 4 ? mq.x >> (8 * k) : (k < 8 ? mq.y >> (8 * (k - 4)) : mq.z);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[8 * k + e] = selb(kb, e, x[8 * k + e]);
        }
      }
      float a = -INFINITY, b = -INFINITY;
#pragma unroll
      for (int e = 0; e < 72; e += 4) {
        a = max3(a, x[e], x[e + 1]);
        b = max3(b, x[e + 2], x[e + 3]);
      }
      return fmaxf(a, b);
    };
    // exp2 and P (bf16) into the P blocks.  The row sum comes out of the PV MMA.
    auto row_exp = [&](const float (&x)[72], float m) {
      const float2 cc = make_float2(c, c), nm = make_float2(-m * c, -m * c);
      const uint32_t rsw = lrow & 7;
      const uint32_t row128 = static_cast<uint32_t>(lrow) * 128, row32 = static_cast<uint32_t>(lrow) * 32;
      const uint32_t sw32 = (lrow >> 2) & 1;
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 4) {
          const int q = 8 * k + e;
          const float2 ya = fma2(make_float2(x[q], x[q + 1]), cc, nm);
          const float2 yb = fma2(make_float2(x[q + 2], x[q + 3]), cc, nm);
          const float2 pa = make_float2(ex2(ya.x), ex2(ya.y));
          const float2 pb = make_float2(ex2(yb.x), ex2(yb.y));
          pk[e / 2] = pack_bf16x2_int(pa.x, pa.y);
          pk[e / 2 + 1] = pack_bf16x2_int(pb.x, pb.y);
        }
        const int g8 = 2 * k + half;   // 16-byte chunk of P along the keys
        uint32_t addr;
        if (k < 8)
          addr = (k < 4 ? pb0 : pb1) + row128 + ((((g8 & 7) ^ rsw)) << 4);
        else
          addr = pb2 + row32 + (((g8 - 16) ^ sw32) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]),
                     "r"(pk[3])
                     : "memory");
      }
    };

    // Iteration `it` does the softmax of tile `it` (if any) and then the epilogue of tile
    // it-1, so the PV MMA of a tile overlaps the next tile's softmax.  One call site each.
    // S is read out of TMEM into registers in one go, so it is released (s_empty) before
    // the exponentials, and the MMA warp can compute the next tile's S underneath them.
    for (long long tile = cta_tile<FUSED>(g, 0);; tile = cta_tile<FUSED>(g, ++it)) {
      const bool have_cur = tile >= 0;
      int head = 0, tok = -1;
      if (have_cur) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
          aborted = true;
          break;
        }
        bool ok = mbar_wait_bounded(table_bar(s), ph, limit_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        head = static_cast<int>(tile) - fdiv(static_cast<int>(tile), g.div_heads) * g.heads;
        const Table& tb = tables[s];
        tok = tb.tok[row];
        const uint4 mq = tb.maskq[my_hi * 2 + half];
        mbar_arrive(empty_bar(s));

        ok = mbar_wait_bounded(s_full, it & 1, limit_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        float x[72];
        const float mh = row_max(x, mq);
        tc_fence_before();
        mbar_arrive(s_empty);   // S of this thread is in registers: the next S may be written
        const int par = it & 1;
        float mrow;
        if (!is_tail) {
          xmax[(par * 2 + half) * 128 + row] = mh;
          mbar_arrive(xmax_bar(par, half));
          ok = mbar_wait_bounded(xmax_bar(par, half ^ 1), (it >> 1) & 1, limit_ns);
          if (!__all_sync(0xffffffffu, ok)) {
            aborted = true;
            break;
          }
          mrow = fmaxf(mh, xmax[(par * 2 + (half ^ 1)) * 128 + row]);
        } else {
          mrow = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
        }
        if (mrow == -INFINITY) mrow = 0.f;
        // P may only be overwritten once the previous tile's PV MMA has consumed it.
        ok = mbar_wait_bounded(is_tail ? p_empty_t : p_empty, par ^ 1, limit_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        row_exp(x, mrow);
        fence_proxy_async_smem();
        mbar_arrive(is_tail ? p_full_t : p_full);
      }
      if (have_prev) {
        if (!epilogue(prev_it, prev_head, prev_tok)) {
          aborted = true;
          break;
        }
      }
      if (!have_cur) break;
      have_prev = true;
      prev_it = it;
      prev_head = head;
      prev_tok = tok;
    }
    if (aborted) {
      if (lane == 0) record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int HD, bool OUT_F32, bool FUSED>
cudaError_t launch_t(const WinGeom& g, const TmaMaps& maps, void* o, int* err, long long limit_ns, int num_sms,
                     const AdalnArgs& fa, cudaStream_t st) {
  auto kern = window_attn_tc_kernel<HD, OUT_F32, FUSED>;
  const int smem = SmemLayout<FUSED>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long units = FUSED ? g.windows : g.windows * g.heads;   // the fused kernel takes whole windows
  const int grid = static_cast<int>(units < num_sms ? units : num_sms);
  kern<<<grid, FUSED ? kThreadsFused : kThreads, smem, st>>>(
      g, maps, o, err, static_cast<unsigned long long>(limit_ns < 0 ? 0 : limit_ns), fa);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn_tc(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                  bool out_f32, int* err, long long spin_limit, int num_sms, cudaStream_t stream) {
  TmaMaps maps;
  const void* ptrs[3] = {q, k, v};
  cudaError_t e = make_maps(g, ptrs, false, &maps);
  if (e != cudaSuccess) return e;
  const AdalnArgs none{};
  if (g.head_dim == 64)
    return out_f32 ? launch_t<64, true, false>(g, maps, o, err, spin_limit, num_sms, none, stream)
                   : launch_t<64, false, false>(g, maps, o, err, spin_limit, num_sms, none, stream);
  return out_f32 ? launch_t<32, true, false>(g, maps, o, err, spin_limit, num_sms, none, stream)
                 : launch_t<32, false, false>(g, maps, o, err, spin_limit, num_sms, none, stream);
}

cudaError_t launch_window_attn_adaln(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                     const AdalnArgs& fa, int* err, long long spin_limit, int num_sms,
                                     cudaStream_t stream) {
  TmaMaps maps;
  const void* ptrs[3] = {q, k, v};
  cudaError_t e = make_maps(g, ptrs, false, &maps);
  if (e != cudaSuccess) return e;
  if (g.head_dim == 64) return launch_t<64, false, true>(g, maps, o, err, spin_limit, num_sms, fa, stream);
  return launch_t<32, false, true>(g, maps, o, err, spin_limit, num_sms, fa, stream);
}

int window_attn_adaln_grid(long long windows, int num_sms) {
  return static_cast<int>(windows < num_sms ? windows : num_sms);
}

}  // namespace s3w
