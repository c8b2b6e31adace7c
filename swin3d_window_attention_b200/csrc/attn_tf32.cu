// Shifted-window attention in the TF32_ACC_FP32 precision mode: FP32 Q/K/V and O, both
// products on the sm_100a tensor cores as tcgen05.mma kind::tf32 with FP32 accumulators in
// TMEM, FP32 softmax.  One persistent CTA per SM, warp-specialised like the BF16 kernel.
//
// Method: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
// section "CuTe DSL window attention" (the two precision modes: TF32_ACC_FP32 takes FP32
// inputs and outputs with TF32 tensor-core MMAs accumulating in FP32, for closer FP32
// fidelity at lower throughput; single-stage path, the whole window's K and V in shared
// memory for N = 144) and section "Mixed-precision inference" (the tf32 backbone tier uses
// this attention with FP32 I/O).  Shift, pad, partition and merge are folded into the
// gather and scatter exactly as in the BF16 kernel (section "Kernel fusion for backbone
// memory traffic").
//
// Differences from the BF16 kernel, all forced by 4-byte operands:
//  * a token row of one head is HD / 32 channel chunks of 128 bytes (32 fp32 each, the
//    swizzle width), so Q, K and V of a tile take 36 KB each at head_dim 64 and two stages
//    fill shared memory;
//  * P (rounded to TF32) is written back by every softmax thread over its own S columns in
//    TMEM (tcgen05.st) and the PV MMA reads its A operand from TMEM, so P needs no shared
//    memory.  S(t+1) overwrites P(t), so the MMA warp issues S(t+1) only once PV(t) has
//    completed; the tile's bytes take twice as long to stream as in BF16, which covers it;
//  * the row sums come from a second MMA chain of P against a block of ones (N = 16) into
//    the 16 TMEM columns after O: the exact normaliser of the TF32 P the PV MMA used.
#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"
#include "s3w_internal.h"
#include "sm100_ptx.cuh"

namespace s3w {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kStagesF = 2;
constexpr int kThreadsF = 384;
constexpr int kMmaWarpF = 9, kTmaWarpF = 10, kTableWarpF = 11, kTailWarpF = 8;

template <int HD>
struct LayoutF {
  static constexpr int kChunks = HD / 32;                    // 128-byte channel chunks per row
  static constexpr int kTensorBytes = kChunks * kChunkTileBytes;
  static constexpr int kStageBytes = 3 * kTensorBytes;       // Q, K, V
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_ONES = OFF_STAGE + kStagesF * kStageBytes;   // 8 key rows x 32 fp32 ones
  static constexpr int OFF_TABLE = OFF_ONES + 1024;
  static constexpr int OFF_SLOTC = OFF_TABLE + kStagesF * kTableBytes;
  static constexpr int OFF_BARS = OFF_SLOTC + kSlotConstBytes;
  // load[2], empty[2], table[2], s_full, p_full, p_full_t, o_full, o_empty, pv_done, drain,
  // row max written[2] (key half)
  static constexpr int kNumBars = 3 * kStagesF + 9;
  static constexpr int OFF_XCHG = OFF_BARS + kNumBars * 8;
  static constexpr int OFF_MISC = OFF_XCHG + 2 * 2 * 128 * 4;
  static constexpr int kSmemBytes = OFF_MISC + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory per CTA");
  static_assert(kStageBytes % 1024 == 0, "stages keep the swizzle atoms aligned");
};

// Shared-memory descriptor layout "128-byte swizzle on a 32-byte base": rows of 128 bytes in
// groups of 4, the four 32-byte chunks of row r permuted by r mod 4.  A 4-byte MN-major
// operand (V here, and the ones block) must be laid out so; the TMA writes V that way
// (CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B).  The plain 128-byte swizzle of 16-byte chunks, right
// for the K-major Q and K, reads as zeros for an MN-major TF32 operand (measured).
constexpr uint32_t kSwizzle128B_Base32B = 1;

// TMEM columns: S0 (rows 0..127) then P0 over it, S1 (tail rows) then P1, O0 and O1 with the
// row sums at column 64 of each.
constexpr uint32_t TF_S0 = 0, TF_S1 = 160, TF_O0 = 320, TF_O1 = 416, TF_SUM = 64;

// Instruction descriptor, kind::tf32: TF32 A and B, FP32 accumulator, dense.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// S = Q K^T over HD in K steps of 8 (32 bytes inside a 128-byte chunk; the next chunk is
// kChunkTileBytes further).  Whole warp executes, `leader` issues.
template <int HD>
__device__ __forceinline__ void umma_tf32_qk(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                             uint32_t leader) {
  constexpr uint64_t kChunkStep = kChunkTileBytes >> 4;
#pragma unroll
  for (int c = 0; c < HD / 32; ++c)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t off = c * kChunkStep + 2 * k;
      const uint32_t acc = (c | k) ? 1u : 0u;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 q, %5, 0;\n\t"
          "@q tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
          "l"(a0 + off), "l"(b0 + off), "r"(idesc), "r"(acc), "r"(leader)
          : "memory");
    }
}

// D (+)= A B with A (TF32, M = 128 x K = 144) in TMEM from column a_tmem, K steps of 8
// columns, and B from shared memory, K steps moving its descriptor by b_step.
__device__ __forceinline__ void umma_tf32_ts_chain(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint64_t b_step,
                                                   uint32_t idesc, uint32_t leader) {
#pragma unroll
  for (int k = 0; k < kN / 8; ++k) {
    const uint32_t acc = k ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem + 8u * k), "l"(b0 + b_step * k), "r"(idesc), "r"(acc), "r"(leader)
        : "memory");
  }
}

// 32 lanes x 32 bits, 8 consecutive columns, registers -> TMEM (thread t: lane base + t).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
// 16 lanes x 32 bits, twice: threads 0..15 -> lanes base + t, columns [c, c + 8); threads
// 16..31 -> lanes base + t - 16, columns [c + 8, c + 16) (the mirror of tmem_ld_16x32bx2_x8).
__device__ __forceinline__ void tmem_st_16x32bx2_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], 8, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// fp32 -> TF32 (round to nearest, ties away from zero), as the 32-bit pattern the MMA reads.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t y;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
  return y;
}

template <int HD, bool OUT_F32>
__global__ void __launch_bounds__(kThreadsF, 1)
window_attn_tf32_kernel(const __grid_constant__ WinGeom g, const __grid_constant__ TmaMaps maps,
                        void* __restrict__ o, int* __restrict__ err, unsigned long long limit_ns) {
  using Lay = LayoutF<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  Table* tables = reinterpret_cast<Table*>(sm + Lay::OFF_TABLE);
  const uint32_t bar0 = sb + Lay::OFF_BARS;
  auto load_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStagesF + s); };
  auto table_bar = [&](int s) { return bar0 + 8u * (2 * kStagesF + s); };
  const uint32_t s_full = bar0 + 8u * (3 * kStagesF + 0);
  const uint32_t p_full = bar0 + 8u * (3 * kStagesF + 1);
  const uint32_t p_full_t = bar0 + 8u * (3 * kStagesF + 2);
  const uint32_t o_full = bar0 + 8u * (3 * kStagesF + 3);
  const uint32_t o_empty = bar0 + 8u * (3 * kStagesF + 4);
  const uint32_t pv_done = bar0 + 8u * (3 * kStagesF + 5);
  const uint32_t drain_bar = bar0 + 8u * (3 * kStagesF + 6);
  auto xmax_bar = [&](int h) { return bar0 + 8u * (3 * kStagesF + 7 + h); };
  float* xmax = reinterpret_cast<float*>(sm + Lay::OFF_XCHG);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 4);
  volatile int* prod_stop = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long num_tiles = g.windows * g.heads;
  const bool has_tail = g.N > 128;
  const uint32_t n_soft = has_tail ? 288u : 256u;

  if (tid == 0) {
    for (int s = 0; s < kStagesF; ++s) {
      mbar_init(load_bar(s), 1);
      mbar_init(empty_bar(s), 1 + n_soft);   // PV commit + every softmax thread (table read)
      mbar_init(table_bar(s), 32);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(p_full_t, 32);
    mbar_init(o_full, 1);
    mbar_init(o_empty, n_soft);
    mbar_init(pv_done, 1);
    mbar_init(drain_bar, 1);
    for (int h = 0; h < 2; ++h) mbar_init(xmax_bar(h), 128);
    *abort_flag = 0;
    *prod_stop = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  SlotConst* slotc = reinterpret_cast<SlotConst*>(sm + Lay::OFF_SLOTC);
  init_slot_consts(g, slotc, tid);
  for (int i = tid; i < 1024 / 16; i += kThreadsF)   // fp32 1.0 = 0x3f800000
    *reinterpret_cast<uint4*>(sm + Lay::OFF_ONES + 16 * i) = make_uint4(0x3f800000u, 0x3f800000u, 0x3f800000u, 0x3f800000u);
  // Slots N..143 are never loaded: keep them zero (finite) for the whole kernel.
  if (g.N < kN) {
    const int per_tile = (kN - g.N) * (kRowBytes / 16);
    for (int i = tid; i < kStagesF * 3 * Lay::kChunks * per_tile; i += kThreadsF) {
      const int chunk16 = i % (kRowBytes / 16);
      const int rest = i / (kRowBytes / 16);
      const int r = g.N + rest % (kN - g.N);
      const int sub = rest / (kN - g.N);   // (stage * 3 + tensor) * chunks + chunk
      *reinterpret_cast<uint4*>(sm + Lay::OFF_STAGE + sub * kChunkTileBytes + r * kRowBytes + chunk16 * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
  }
  fence_proxy_async_smem();
  if (warp == kMmaWarpF) {
    tmem_alloc(sb + Lay::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ring ring{sb + Lay::OFF_STAGE, load_bar(0), empty_bar(0), table_bar(0)};

  if (warp == kTmaWarpF) {
    if (lane == 0)
      tma_loader<Lay::kChunks, 32, kStagesF, Lay::kStageBytes>(g, maps, ring, HD, num_tiles, abort_flag, err,
                                                               limit_ns);
  } else if (warp == kTableWarpF) {
    table_writer<kStagesF>(g, tables, slotc, ring, num_tiles, abort_flag, prod_stop, err, limit_ns, lane);
  } else if (warp == kMmaWarpF) {
    // ------------------------------------------------------------------ MMA issuer
    // Per tile t: PV(t) (and its row sums) once P(t) is in TMEM and O is free, then S(t+1)
    // once PV(t) has completed (S(t+1) overwrites P(t)).
    constexpr uint32_t idesc_s = idesc_tf32_f32(128, kN, false, false);
    constexpr uint32_t idesc_o = idesc_tf32_f32(128, HD, false, true);
    constexpr uint32_t idesc_l = idesc_tf32_f32(128, 16, false, true);
    // Q / K of stage 0: K-major, 128B swizzle, 8-row atoms 1024 bytes apart
    const uint64_t dq0 = smem_desc(sb + Lay::OFF_STAGE, 16, 1024, kSwizzle128B);
    constexpr uint64_t kTensorStep = Lay::kTensorBytes >> 4;
    // V of stage 0: MN-major, 128B swizzle on a 32B base; 4 keys x 32 channels per atom (512
    // bytes apart along the keys), the next 32 channels one chunk further (leading byte
    // offset); a K step of 8 keys moves 1024 bytes
    const uint64_t dv0 =
        smem_desc(sb + Lay::OFF_STAGE + 2 * Lay::kTensorBytes, kChunkTileBytes, 512, kSwizzle128B_Base32B);
    const uint64_t dones = smem_desc(sb + Lay::OFF_ONES, 1024, 512, kSwizzle128B_Base32B);
    constexpr uint64_t kStageStep = Lay::kStageBytes >> 4;
    const uint32_t leader = lane == 0 ? 1u : 0u;
    bool issued = false;
    auto issue_s = [&](int jt) -> bool {
      const int s = jt % kStagesF;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(load_bar(s), (jt / kStagesF) & 1, limit_ns))) return false;
      if (jt > 0 && !__all_sync(0xffffffffu, mbar_wait_bounded(pv_done, (jt - 1) & 1, limit_ns))) return false;
      fence_proxy_async_smem();
      tc_fence_after();
      const uint64_t qd = dq0 + s * kStageStep, kd = qd + kTensorStep;
      umma_tf32_qk<HD>(tmem + TF_S0, qd, kd, idesc_s, leader);
      if (has_tail) umma_tf32_qk<HD>(tmem + TF_S1, qd + ((128 * kRowBytes) >> 4), kd, idesc_s, leader);
      umma_commit_leader(s_full, leader);
      issued = true;
      return true;
    };
    auto issue_pv = [&](int jt) -> bool {
      const int s = jt % kStagesF;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full, jt & 1, limit_ns))) return false;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_empty, (jt & 1) ^ 1, limit_ns))) return false;
      tc_fence_after();
      const uint64_t vd = dv0 + s * kStageStep;
      umma_tf32_ts_chain(tmem + TF_O0, tmem + TF_S0, vd, 1024 >> 4, idesc_o, leader);
      umma_tf32_ts_chain(tmem + TF_O0 + TF_SUM, tmem + TF_S0, dones, 0, idesc_l, leader);
      if (has_tail) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full_t, jt & 1, limit_ns))) return false;
        tc_fence_after();
        umma_tf32_ts_chain(tmem + TF_O1, tmem + TF_S1, vd, 1024 >> 4, idesc_o, leader);
        umma_tf32_ts_chain(tmem + TF_O1 + TF_SUM, tmem + TF_S1, dones, 0, idesc_l, leader);
      }
      umma_commit_leader(o_full, leader);
      umma_commit_leader(empty_bar(s), leader);
      umma_commit_leader(pv_done, leader);
      return true;
    };
    bool ok = !g.test_stall || __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, limit_ns));
    const long long my_tiles =
        static_cast<long long>(blockIdx.x) < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (ok && my_tiles > 0) ok = issue_s(0);
    for (long long t = 0; ok && t < my_tiles; ++t) {
      ok = !__any_sync(0xffffffffu, *abort_flag != 0);
      if (ok) ok = issue_pv(static_cast<int>(t));
      if (ok && t + 1 < my_tiles) ok = issue_s(static_cast<int>(t + 1));
    }
    if (!ok && lane == 0) {
      record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
    if (lane == 0 && issued) {
      umma_commit(drain_bar);
      if (!mbar_wait_bounded(drain_bar, 0, 2000000000ull)) record_error(err, kStatusTimeout);
    }
    __syncwarp();
  } else if (warp < 8 || (warp == kTailWarpF && has_tail)) {
    // ------------------------------------------------------------------ softmax + epilogue
    // Thread roles as in the BF16 kernel: main warp w owns row 32 (w % 4) + lane of S0 and
    // the key half w / 4 (key groups 2k + half, 72 keys); tail warp 8 owns row 128 + lane % 16
    // of S1, half lane / 16.  P goes back over the same TMEM columns the logits came from.
    const bool is_tail = warp == kTailWarpF;
    const float c = g.scale_log2;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int half = is_tail ? (lane >> 4) : ((warp >> 2) & 1);
    const int row = is_tail ? 128 + (lane & 15) : (warp & 3) * 32 + lane;
    const uint32_t s_base = is_tail ? tmem + TF_S1 : tmem + lane_base + TF_S0 + 8 * half;
    const uint32_t o_base = is_tail ? tmem + TF_O1 : tmem + lane_base + TF_O0 + 16 * half;
    const uint32_t my_hi = [&] {
      uint32_t h = 0;
#pragma unroll
      for (int a = 0; a < 3; ++a) h |= ((slotc->hi[a][row >> 5] >> (row & 31)) & 1u) << a;
      return h;
    }();
    int it = 0;
    bool have_prev = false;
    int prev_it = 0, prev_head = 0, prev_tok = -1;
    bool aborted = false;

    // Epilogue of a finished tile: this thread's O columns (groups of 16: 32m + 16 half) and
    // the row sum from TMEM, scaled by 1/rowsum, stored to the query's grid position.
    auto epilogue = [&](int pit, int head, int tok) -> bool {
      bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_full, pit & 1, limit_ns));
      if (!ok) return false;
      tc_fence_after();
      float ov[(HD + 31) / 32 * 16];
      float l;
      if (!is_tail) {
#pragma unroll
        for (int m = 0; m < (HD + 31) / 32; ++m) tmem_ld16(o_base + 32 * m, ov + 16 * m);
        tmem_ld1(o_base - 16 * half + TF_SUM, &l);
      } else {
#pragma unroll
        for (int m = 0; m < (HD + 31) / 32; ++m) tmem_ld_16x32bx2_x16(o_base + 32 * m, ov + 16 * m);
        tmem_ld_16x32bx2_x1(o_base + TF_SUM, &l);
      }
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < (HD + 31) / 32; ++m) reg_fence16(ov + 16 * m);
      reg_fence1(&l);
      tc_fence_before();
      mbar_arrive(o_empty);
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      store_o_row<HD, OUT_F32>(o, g.o_stride, g.o_rows_32b != 0, tok, head, half, lane, ov, inv);
      return true;
    };

    auto selb = [](uint32_t w, int e, float x) { return ((w >> e) & 1u) ? x : -INFINITY; };
    for (long long tile = blockIdx.x;; tile += gridDim.x, ++it) {
      const bool have_cur = tile < num_tiles;
      int head = 0, tok = -1;
      if (have_cur) {
        const int s = it % kStagesF;
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
          aborted = true;
          break;
        }
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(table_bar(s), (it / kStagesF) & 1, limit_ns))) {
          aborted = true;
          break;
        }
        head = static_cast<int>(tile) - fdiv(static_cast<int>(tile), g.div_heads) * g.heads;
        const Table& tb = tables[s];
        tok = tb.tok[row];
        const uint4 mq = tb.maskq[my_hi * 2 + half];
        mbar_arrive(empty_bar(s));
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full, it & 1, limit_ns))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        // the thread's 72 logits: key groups 2k + half of 8 keys, column 16k + 8 half
        float x[72];
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
        const float mh = fmaxf(a, b);
        const int par = it & 1;
        float mrow;
        if (!is_tail) {
          xmax[(par * 2 + half) * 128 + row] = mh;
          mbar_arrive(xmax_bar(half));
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(xmax_bar(half ^ 1), par, limit_ns))) {
            aborted = true;
            break;
          }
          mrow = fmaxf(mh, xmax[(par * 2 + (half ^ 1)) * 128 + row]);
        } else {
          mrow = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
        }
        if (mrow == -INFINITY) mrow = 0.f;
        // P = exp2(c (x - m)) rounded to TF32, over the logits' own TMEM columns
        const float2 cc = make_float2(c, c), nm = make_float2(-mrow * c, -mrow * c);
#pragma unroll
        for (int k = 0; k < 9; ++k) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 y = fma2(make_float2(x[8 * k + e], x[8 * k + e + 1]), cc, nm);
            pk[e] = to_tf32(ex2(y.x));
            pk[e + 1] = to_tf32(ex2(y.y));
          }
          if (!is_tail)
            tmem_st8(s_base + 16 * k, pk);
          else
            tmem_st_16x32bx2_x8(s_base + 16 * k, pk);
        }
        tmem_wait_st();
        tc_fence_before();
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
  if (warp == kMmaWarpF) tmem_dealloc(tmem, 512);
}

template <int HD, bool OUT_F32>
cudaError_t launch_f(const WinGeom& g, const TmaMaps& maps, void* o, int* err, long long limit_ns, int num_sms,
                     cudaStream_t st) {
  auto kern = window_attn_tf32_kernel<HD, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LayoutF<HD>::kSmemAlloc);
  if (e != cudaSuccess) return e;
  const long long tiles = g.windows * g.heads;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, kThreadsF, LayoutF<HD>::kSmemAlloc, st>>>(g, maps, o, err,
                                                          static_cast<unsigned long long>(limit_ns < 0 ? 0 : limit_ns));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn_tf32(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                    bool out_f32, int* err, long long spin_limit, int num_sms, cudaStream_t stream) {
  TmaMaps maps;
  const void* ptrs[3] = {q, k, v};
  cudaError_t e = make_maps(g, ptrs, true, &maps, /*v_atom32=*/true);
  if (e != cudaSuccess) return e;
  if (g.head_dim == 64)
    return out_f32 ? launch_f<64, true>(g, maps, o, err, spin_limit, num_sms, stream)
                   : launch_f<64, false>(g, maps, o, err, spin_limit, num_sms, stream);
  return out_f32 ? launch_f<32, true>(g, maps, o, err, spin_limit, num_sms, stream)
                 : launch_f<32, false>(g, maps, o, err, spin_limit, num_sms, stream);
}

}  // namespace s3w
