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
//                      output column, see below), scales by 1/rowsum and stores them to the
//                      query's original grid position; padded slots are dropped.
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
//   TMA warp 10        one thread loads the tile's Q, K and V with TMA: one box per T-slab
//                      of the window (win_h x win_w tokens) per tensor, cut where the window
//                      wraps around a seam of the shifted grid, straight from grid layout into
//                      a 3-stage ring in the tensor core's 128-byte swizzled K-major layout;
//                      padded coordinates are out of bounds and read as zero.  It runs ahead
//                      as far as the ring allows.
//   table warp 11      writes the slot -> grid-token table, a bitmask of the real slots, the
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

constexpr int kStages = 3;
constexpr int kTileBytes = kChunkTileBytes;         // 18432: one of Q / K / V (one head = 128 B rows)
constexpr int kStageBytes = 3 * kTileBytes;         // 55296

// Shared-memory map (offsets from a 1024-byte aligned base).
// Once S = Q K^T of a tile has been computed, its Q and K tiles are dead: the P of the 128
// main rows (36 KB, exactly the size of Q + K) is written over them, in the tile's own
// stage, so P of the next tile never waits for the PV MMA of this one.  In a stage:
//   P rows 0..127, keys 0..63    at +0      (128B swizzle, over Q)
//   P rows 0..127, keys 64..127  at +16384  (128B swizzle, over Q rows 128.. and K)
//   P rows 0..127, keys 128..143 at +32768  (32B swizzle, 4 KB, over K)
// The 16 tail rows' P of stage s lives in a block of its own at s * kTailPBytes.  Their
// M = 128 descriptors also cover rows 16..127, which fall on the blocks and stages that
// follow (valid memory; the results of those rows are never used).
constexpr int kTailPBytes = 5120;
constexpr int OFF_P1B0 = 0;        // tail P rows 0..15, keys 0..63   (128B swizzle)
constexpr int OFF_P1B1 = 2048;     // tail P rows 0..15, keys 64..127 (128B swizzle)
constexpr int OFF_P1B2 = 4096;     // tail P rows 0..15, keys 128..143 (32B swizzle)
constexpr int OFF_P0B0 = 0;        // main P, relative to the stage
constexpr int OFF_P0B1 = 16384;
constexpr int OFF_P0B2 = 32768;
static_assert(OFF_P0B2 + 128 * 32 <= 2 * kTileBytes, "main P fits over Q and K");
constexpr int OFF_STAGE = kStages * kTailPBytes;   // 15360 (1024-aligned)
static_assert(OFF_STAGE % 1024 == 0 && kStageBytes % 1024 == 0, "swizzle atoms stay aligned");
static_assert((kStages - 1) * kTailPBytes + 128 * kRowBytes <= OFF_STAGE + kStageBytes,
              "the tail P descriptors' unused rows stay inside the stages");
// 16 key rows of bf16 ones in the V operand's layout: the PV MMA reads them as 16 more
// output columns (through the descriptor's leading byte offset), so every such column of O
// is the row sum of P as rounded to bf16, the exact normaliser of the P the MMA used.
constexpr int OFF_ONES = OFF_STAGE + kStages * kStageBytes;
constexpr int kOnesBytes = 16 * kRowBytes;
constexpr int OFF_TABLE = OFF_ONES + kOnesBytes;

constexpr int OFF_SLOTC = OFF_TABLE + kStages * kTableBytes;
constexpr int OFF_BARS = OFF_SLOTC + kSlotConstBytes;
// barriers: load[3] (TMA bytes), empty[3], table[3], s_full, s_empty, p_full[2] (tile
// parity), o_full, o_empty, drain, row max written[2][2] (tile parity, key half), tail
// p_full[2] (tile parity).
// P and the row maxima of a tile are handed over on barriers of the tile's parity.  Nothing
// stops one softmax warp from arriving for tile t+1 before another has arrived for tile t,
// or the tail warp from completing tile t+1's P before the MMA warp has waited for tile
// t's; but no warp can arrive for tile t+2 before every waiter of tile t has passed (that
// needs S(t+2), which the MMA warp issues only after its waits of tile t).
constexpr int kNumBars = 3 * kStages + 13;
// Row max of each key half of the main rows, exchanged between the two warps that share a
// row: [tile parity][key half][row].
constexpr int OFF_XCHG = OFF_BARS + kNumBars * 8;
constexpr int kXchgFloats = 2 * 2 * 128;
constexpr int OFF_MISC = OFF_XCHG + kXchgFloats * 4;   // tmem address, abort flag, producer stop
constexpr int kSmemBytes = OFF_MISC + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;       // slack for the 1024-byte alignment
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");

// TMEM columns (fp32 accumulators, lane = row).  Every MMA destination is 32-aligned.  O
// has 80 columns: the head's outputs (the first head_dim of 64), then from column 64 on 16
// copies of the row sum.
constexpr uint32_t TM_S0 = 0, TM_S1 = 160, TM_O0 = 320, TM_O1 = 416;
constexpr uint32_t kOnesCol = 64;
constexpr uint32_t kTmemCols = 512;

constexpr int kThreads = 512;
constexpr int kMainWarps = 8;          // rows 0..127: warp w holds lanes 32 (w % 4) .., keys 72 (w / 4) ..
constexpr int kTailWarp = 8;           // tail rows 128..143 (TMEM lane quarter 0, like warp 0)
constexpr int kMmaWarp = 9;
constexpr int kTmaWarp = 10;
constexpr int kFirstProducerWarp = 11;
constexpr int kProducerThreads = 32;   // table writer (warp 11)
constexpr int kFirstEpiWarp = 12;      // warps 12..15: O of TMEM lane quarter warp % 4 to global memory
constexpr int kEpiThreads = 128;

// Operand descriptors.  K-major 128B swizzle: 8-row x 128-byte atoms, 1024 bytes apart.
// K-major 32B swizzle: 8-row x 32-byte atoms, 256 bytes apart.  MN-major 128B swizzle (V,
// whose rows are keys = the K dimension): 8-key x 64-element atoms, 1024 bytes apart along
// K; the leading byte offset is the distance to the next 64 elements along N.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128B); }
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t addr) { return smem_desc(addr, 16, 256, kSwizzle32B); }

template <int HD, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
window_attn_tc_kernel(const __grid_constant__ WinGeom g, const __grid_constant__ TmaMaps maps,
                      void* __restrict__ o, int* __restrict__ err, unsigned long long limit_ns) {
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
  auto p_full = [&](int par) { return bar0 + 8u * (3 * kStages + 2 + par); };   // main-row P of a tile
  const uint32_t o_full = bar0 + 8u * (3 * kStages + 4);
  const uint32_t o_empty = bar0 + 8u * (3 * kStages + 5);
  const uint32_t drain_bar = bar0 + 8u * (3 * kStages + 6);
  // key half h of a tile of parity par wrote its row maxima
  auto xmax_bar = [&](int par, int h) { return bar0 + 8u * (3 * kStages + 7 + 2 * par + h); };
  // P of the main rows and of the tail rows are handed over separately, so the main rows'
  // PV MMA need not wait for the tail warp.
  auto p_full_t = [&](int par) { return bar0 + 8u * (3 * kStages + 11 + par); };
  float* xmax = reinterpret_cast<float*>(sm + OFF_XCHG);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* prod_stop = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long num_tiles = g.windows * g.heads;
  const bool has_tail = g.N > 128;
  const uint32_t n_soft = has_tail ? 288u : 256u;   // softmax threads: main rows (+ tail warp)

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(load_bar(s), 1);                        // the TMA thread's expect_tx arrival + bytes
      mbar_init(empty_bar(s), 1 + n_soft + kEpiThreads);  // PV commit + softmax and epilogue threads (table read)
      mbar_init(table_bar(s), kProducerThreads);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, n_soft);
    for (int par = 0; par < 2; ++par) mbar_init(p_full(par), 256);
    for (int par = 0; par < 2; ++par) mbar_init(p_full_t(par), 32);
    mbar_init(o_full, 1);
    mbar_init(o_empty, kEpiThreads);
    mbar_init(drain_bar, 1);
    for (int par = 0; par < 2; ++par)
      for (int h = 0; h < 2; ++h) mbar_init(xmax_bar(par, h), 128);
    *abort_flag = 0;
    *prod_stop = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  SlotConst* slotc = reinterpret_cast<SlotConst*>(sm + OFF_SLOTC);
  init_slot_consts(g, slotc, tid);
  for (int i = tid; i < kOnesBytes / 16; i += kThreads)   // bf16 1.0 = 0x3f80
    *reinterpret_cast<uint4*>(sm + OFF_ONES + 16 * i) = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  fence_proxy_async_smem();
  // Slots N..143 are never loaded: keep them zero (finite) for the whole kernel.
  if (g.N < kN) {
    for (int i = tid; i < kStages * 3 * (kN - g.N) * (kRowBytes / 16); i += kThreads) {
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
    // ------------------------------------------------------------------ TMA loads
    if (lane == 0) tma_loader<1, 64, kStages, kStageBytes>(g, maps, ring, HD, num_tiles, abort_flag, err, limit_ns);
  } else if (warp == kFirstProducerWarp) {
    // ------------------------------------------------------------------ tile tables
    table_writer<kStages>(g, tables, slotc, ring, num_tiles, abort_flag, prod_stop, err, limit_ns, lane);
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
    // P of the main rows over Q and K of stage 0; the tail rows' P block of stage 0
    const uint64_t dp0 = desc_kmajor_sw128(sb + OFF_STAGE + OFF_P0B0);
    const uint64_t dp0b = desc_kmajor_sw32(sb + OFF_STAGE + OFF_P0B2);
    const uint64_t dp1 = desc_kmajor_sw128(sb + OFF_P1B0), dp1b = desc_kmajor_sw32(sb + OFF_P1B2);
    constexpr uint64_t kStageStep = kStageBytes >> 4;
    constexpr uint64_t kTailStep = kTailPBytes >> 4;
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
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full(jt & 1), (jt >> 1) & 1, limit_ns))) return false;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_empty, (jt & 1) ^ 1, limit_ns))) return false;
      tc_fence_after();
      // Moving V by d (bytes / 16) moves the ones block's leading offset by -d.
      const uint64_t dstage = s * kStageStep;
      const uint64_t vd = dv0 + dstage - (dstage << 16);
      umma_chain_pv(tmem + TM_O0, dp0 + dstage, vd, idesc_o, leader, dp0b + dstage, ((OFF_P0B1 - OFF_P0B0) >> 4) - 6);
      if (has_tail) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full_t(jt & 1), (jt >> 1) & 1, limit_ns))) return false;
        tc_fence_after();
        const uint64_t dtail = s * kTailStep;
        umma_chain_pv(tmem + TM_O1, dp1 + dtail, vd, idesc_o, leader, dp1b + dtail,
                      ((OFF_P1B1 - OFF_P1B0) >> 4) - 6);
      }
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
    const long long my_tiles =
        static_cast<long long>(blockIdx.x) < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
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
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------------ epilogue
    // Warp 12 + q reads TMEM lane quarter q of O0 (query rows 32q .. 32q + 31, one row per
    // thread: the head's columns and the row sum, an MMA output column), releases O, scales
    // by 1/rowsum and stores each row to its query's original grid position; padded slots are
    // dropped.  Warp 12 also takes the 16 tail rows of O1 (TMEM lanes 0..15), half a row per
    // thread (16x32bx2 shape).  The grid tokens are read from the tile's table before the
    // stage is released.
    const int q = warp - kFirstEpiWarp;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int row = q * 32 + lane;
    const bool do_tail = has_tail && q == 0;
    const int thalf = lane >> 4;
    auto store16 = [&](int tk, int head, int col, const float* vals, float scl) {
      // 16 consecutive outputs of one row starting at column `col`
      if constexpr (OUT_F32) {
        float* dst = static_cast<float*>(o) + static_cast<long long>(tk) * g.o_stride + head * HD + col;
#pragma unroll
        for (int h8 = 0; h8 < 16; h8 += 8) {
          if (g.o_rows_32b) {
            uint32_t u[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] = __float_as_uint(vals[h8 + e] * scl);
            st_global_v8(dst + h8, u);
          } else {
#pragma unroll
            for (int e = 0; e < 8; e += 4)
              *reinterpret_cast<float4*>(dst + h8 + e) =
                  make_float4(vals[h8 + e] * scl, vals[h8 + e + 1] * scl, vals[h8 + e + 2] * scl, vals[h8 + e + 3] * scl);
          }
        }
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o) + static_cast<long long>(tk) * g.o_stride + head * HD + col;
        uint32_t u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) u[e] = pack_bf16x2_rne_int(vals[2 * e] * scl, vals[2 * e + 1] * scl);
        if (g.o_rows_32b) {
          st_global_v8(dst, u);
        } else {
          *reinterpret_cast<uint4*>(dst) = make_uint4(u[0], u[1], u[2], u[3]);
          *reinterpret_cast<uint4*>(dst + 8) = make_uint4(u[4], u[5], u[6], u[7]);
        }
      }
    };
    int it = 0;
    bool aborted = false;
    for (long long tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int s = it % kStages;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        aborted = true;
        break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(table_bar(s), (it / kStages) & 1, limit_ns))) {
        aborted = true;
        break;
      }
      const int tok = tables[s].tok[row];
      const int tok_t = do_tail ? tables[s].tok[128 + (lane & 15)] : -1;
      mbar_arrive(empty_bar(s));
      const int head = static_cast<int>(tile) - fdiv(static_cast<int>(tile), g.div_heads) * g.heads;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_full, it & 1, limit_ns))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float ov[HD], l;
      float ot[HD / 2], lt = 0.f;
#pragma unroll
      for (int m = 0; m < HD / 16; ++m) tmem_ld16(tmem + lane_base + TM_O0 + 16 * m, ov + 16 * m);
      tmem_ld1(tmem + lane_base + TM_O0 + kOnesCol, &l);
      if (do_tail) {
#pragma unroll
        for (int m = 0; m < HD / 32; ++m) tmem_ld_16x32bx2_x16(tmem + TM_O1 + 32 * m, ot + 16 * m);
        tmem_ld_16x32bx2_x1(tmem + TM_O1 + kOnesCol, &lt);
      }
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < HD / 16; ++m) reg_fence16(ov + 16 * m);
      reg_fence1(&l);
      if (do_tail) {
#pragma unroll
        for (int m = 0; m < HD / 32; ++m) reg_fence16(ot + 16 * m);
        reg_fence1(&lt);
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      if (tok >= 0) {
        const float inv = l > 0.f ? rcp_approx(l) : 0.f;
#pragma unroll
        for (int m = 0; m < HD / 16; ++m) store16(tok, head, 16 * m, ov + 16 * m, inv);
      }
      if (tok_t >= 0) {
        const float inv = lt > 0.f ? rcp_approx(lt) : 0.f;
#pragma unroll
        for (int m = 0; m < HD / 32; ++m) store16(tok_t, head, 32 * m + 16 * thalf, ot + 16 * m, inv);
      }
    }
    if (aborted) {
      if (lane == 0) record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  } else if (warp < kMainWarps || (warp == kTailWarp && has_tail)) {
    // ------------------------------------------------------------------ softmax
    // Every softmax thread owns one (query row, key half) and runs the same code.  Half h
    // holds the key groups 2k + h (k = 0..8) of 8 keys each, 72 keys.  Main warp w: row
    // 32 (w % 4) + lane (its TMEM lane in S0 = Q[0:128] K^T), half w / 4, read with the
    // 32x32b shape at column 16k + 8h; its partner (same row, other half) is warp w ^ 4,
    // and the two swap row maxima through shared memory.  Tail warp 8: row 128 + lane % 16
    // (TMEM lane lane % 16 of S1 = Q[128:144] K^T), half lane / 16, read with the 16x32bx2
    // shape (threads 16..31 see the columns 8 further on); its partner is lane ^ 16 of the
    // same warp (a shuffle).
    const bool is_tail = warp == kTailWarp;
    const float c = g.scale_log2;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int half = is_tail ? (lane >> 4) : ((warp >> 2) & 1);
    const int row = is_tail ? 128 + (lane & 15) : (warp & 3) * 32 + lane;
    const int lrow = is_tail ? (lane & 15) : row;   // row inside its P blocks
    // P blocks of stage 0 (main rows: over that stage's Q and K; tail rows: its tail block)
    const uint32_t pb0 = sb + (is_tail ? OFF_P1B0 : OFF_STAGE + OFF_P0B0);
    const uint32_t pb1 = sb + (is_tail ? OFF_P1B1 : OFF_STAGE + OFF_P0B1);
    const uint32_t pb2 = sb + (is_tail ? OFF_P1B2 : OFF_STAGE + OFF_P0B2);
    const uint32_t p_stage_step = is_tail ? kTailPBytes : kStageBytes;
    const uint32_t s_base = is_tail ? tmem + TM_S1 : tmem + lane_base + TM_S0 + 8 * half;
    const uint32_t my_hi = [&] {
      uint32_t h = 0;
#pragma unroll
      for (int a = 0; a < 3; ++a) h |= ((slotc->hi[a][row >> 5] >> (row & 31)) & 1u) << a;
      return h;
    }();
    int it = 0;
    bool aborted = false;

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
    auto row_exp = [&](const float (&x)[72], float m, uint32_t pofs) {
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
          addr = (k < 4 ? pb0 : pb1) + pofs + row128 + ((((g8 & 7) ^ rsw)) << 4);
        else
          addr = pb2 + pofs + row32 + (((g8 - 16) ^ sw32) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]),
                     "r"(pk[3])
                     : "memory");
      }
    };

    // S is read out of TMEM into registers in one go, so it is released (s_empty) before
    // the exponentials, and the MMA warp can compute the next tile's S underneath them.
    for (long long tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
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
      const uint4 mq = tables[s].maskq[my_hi * 2 + half];
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
      // P goes to the tile's own stage (over its Q and K, consumed by S, which s_full
      // guaranteed above): no wait for the previous tile's PV.
      row_exp(x, mrow, static_cast<uint32_t>(s) * p_stage_step);
      fence_proxy_async_smem();
      mbar_arrive(is_tail ? p_full_t(par) : p_full(par));
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

template <int HD, bool OUT_F32>
cudaError_t launch_t(const WinGeom& g, const TmaMaps& maps, void* o, int* err, long long limit_ns, int num_sms,
                     cudaStream_t st) {
  auto kern = window_attn_tc_kernel<HD, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  const long long tiles = g.windows * g.heads;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, kThreads, kSmemAlloc, st>>>(g, maps, o, err, static_cast<unsigned long long>(limit_ns < 0 ? 0 : limit_ns));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn_tc(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                  bool out_f32, int* err, long long spin_limit, int num_sms, cudaStream_t stream) {
  TmaMaps maps;
  const void* ptrs[3] = {q, k, v};
  cudaError_t e = make_maps(g, ptrs, false, &maps);
  if (e != cudaSuccess) return e;
  if (g.head_dim == 64)
    return out_f32 ? launch_t<64, true>(g, maps, o, err, spin_limit, num_sms, stream)
                   : launch_t<64, false>(g, maps, o, err, spin_limit, num_sms, stream);
  return out_f32 ? launch_t<32, true>(g, maps, o, err, spin_limit, num_sms, stream)
                 : launch_t<32, false>(g, maps, o, err, spin_limit, num_sms, stream);
}

}  // namespace s3w
