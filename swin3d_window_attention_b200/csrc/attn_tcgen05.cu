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
// Work unit ("tile"): one (sample, window, head).  Per tile:
//   producer warps 5-7  gather 3 x 144 token rows (16-byte cp.async, zero-fill for padded
//                       slots) into a 3-stage shared-memory ring laid out as the 128-byte
//                       swizzled operand layout of the tensor core; compute the slot ->
//                       grid-token table, the Swin region label of every slot and one
//                       key bitmask per label.
//   MMA warp 4          S0 = Q[0:128] K^T and S1 = Q[128:144] K^T (M = 128, N = 144,
//                       K = head_dim) into TMEM; after softmax, O0 = P0 V and O1 = P1 V
//                       (M = 128, N = head_dim, K = 144, V read as an MN-major operand).
//   softmax warps 0-3   thread t owns TMEM lane t = query row t: load the S row (144 fp32),
//                       mask by region label / padding, exact row max, exp2, row sum, round
//                       P to bf16 into shared memory; warp 0 also handles the 16 tail rows.
//                       Then (one tile later, so the PV MMA overlaps the next softmax) load
//                       the O row, scale by 1/rowsum, and store it to the query's original
//                       grid position (padded slots are dropped).
// Synchronisation is by mbarriers only; every wait is bounded by a time limit and a
// timeout unwinds the whole CTA (error word set, copies drained, TMEM freed).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s3w_internal.h"
#include "sm100_ptx.cuh"

namespace s3w {
namespace {

using namespace sm100;

constexpr int kN = 144;          // tokens per window slot block (queries and keys)
constexpr int kStages = 3;
constexpr int kRowBytes = 128;   // one token row of one head in shared memory (swizzle width)
constexpr int kTileBytes = kN * kRowBytes;          // 18432: one of Q / K / V
constexpr int kStageBytes = 3 * kTileBytes;         // 55296
constexpr int kLabels = 28;      // 27 region labels + "padded"
constexpr int kPadLabel = 27;
constexpr int kMaskWords = 5;    // 144 key bits

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr int OFF_P1B0 = 0;        // tail P rows 0..15, keys 0..63   (128B swizzle)
constexpr int OFF_P1B1 = 2048;     // tail P rows 0..15, keys 64..127 (128B swizzle)
constexpr int OFF_P1B2 = 4096;     // tail P rows 0..15, keys 128..143 (32B swizzle)
constexpr int OFF_P0B0 = 5120;     // P rows 0..127, keys 0..63
constexpr int OFF_P0B1 = OFF_P0B0 + 16384;
constexpr int OFF_P0B2 = OFF_P0B1 + 16384;   // keys 128..143, 32B swizzle, 4 KB
constexpr int OFF_STAGE = OFF_P0B2 + 4096;   // 41984 (1024-aligned)
constexpr int OFF_TABLE = OFF_STAGE + kStages * kStageBytes;

struct Table {
  int tok[kN];                       // flat grid token of each slot, -1 = padded
  uint32_t mask[kLabels * kMaskWords];
  uint8_t lab[kN];                   // region label of each slot (kPadLabel = padded)
};
constexpr int kTableBytes = (static_cast<int>(sizeof(Table)) + 15) & ~15;
constexpr int OFF_BARS = OFF_TABLE + kStages * kTableBytes;
// barriers: full[3], empty[3], s_full, s_empty, p_full, p_empty, o_full, o_empty, drain
constexpr int kNumBars = 2 * kStages + 7;
constexpr int OFF_MISC = OFF_BARS + kNumBars * 8;   // tmem address, abort flag, producer stop
constexpr int kSmemBytes = OFF_MISC + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;       // slack for the 1024-byte alignment

// TMEM columns (fp32 accumulators, lane = row).  Every MMA destination is 32-aligned.
constexpr uint32_t TM_S0 = 0, TM_S1 = 160, TM_O0 = 320, TM_O1 = 384;
constexpr uint32_t kTmemCols = 512;

constexpr int kThreads = 256;
constexpr int kProducerThreads = 96;

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Descriptors of the A/B operands (see the layout notes at the top of the file).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128B); }
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t addr) { return smem_desc(addr, 16, 256, kSwizzle32B); }
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t addr) { return smem_desc(addr, 16, 1024, kSwizzle128B); }

template <int HD, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
window_attn_tc_kernel(const __grid_constant__ WinGeom g, const __nv_bfloat16* __restrict__ q,
                      const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                      void* __restrict__ o, int* __restrict__ err, unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  Table* tables = reinterpret_cast<Table*>(sm + OFF_TABLE);
  const uint32_t bar0 = sb + OFF_BARS;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t s_full = bar0 + 8u * (2 * kStages + 0);
  const uint32_t s_empty = bar0 + 8u * (2 * kStages + 1);
  const uint32_t p_full = bar0 + 8u * (2 * kStages + 2);
  const uint32_t p_empty = bar0 + 8u * (2 * kStages + 3);
  const uint32_t o_full = bar0 + 8u * (2 * kStages + 4);
  const uint32_t o_empty = bar0 + 8u * (2 * kStages + 5);
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 6);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* prod_stop = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long num_tiles = g.windows * g.heads;
  const bool has_tail = g.N > 128;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), kProducerThreads);
      mbar_init(empty_bar(s), 1 + 128);   // PV commit + every softmax thread (table read)
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 128);
    mbar_init(p_full, 128);
    mbar_init(p_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 128);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *prod_stop = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 4) {
    tmem_alloc(sb + OFF_MISC, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 5) {
    // ------------------------------------------------------------------ producers
    const int p = tid - 160;
    constexpr int CH = HD / 8;                   // 16-byte chunks per head row
    int it = 0;
    bool stopped = false;
    for (long long tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      if (p == 0) {
        const bool ok = mbar_wait_bounded(empty_bar(s), ph ^ 1, limit_ns);
        if (!ok) {
          record_error(err, kStatusTimeout);
          *abort_flag = 1;
        }
        *prod_stop = (!ok || *abort_flag) ? 1 : 0;
      }
      named_bar_sync(1, kProducerThreads);
      if (*prod_stop) {
        stopped = true;
        break;
      }
      const long long win = tile / g.heads;
      const int head = static_cast<int>(tile - win * g.heads);
      Table& tb = tables[s];
      for (int r = p; r < kN; r += kProducerThreads) {
        int lab = kPadLabel;
        long long tk = -1;
        if (r < g.N) {
          int l2;
          tk = slot_token(g, win, r, &l2);
          if (tk >= 0) lab = l2;
        }
        tb.tok[r] = static_cast<int>(tk);
        tb.lab[r] = static_cast<uint8_t>(lab);
      }
      for (int w = p; w < kLabels * kMaskWords; w += kProducerThreads) tb.mask[w] = 0u;
      named_bar_sync(1, kProducerThreads);
      for (int r = p; r < kN; r += kProducerThreads)
        atomicOr(&tb.mask[tb.lab[r] * kMaskWords + (r >> 5)], 1u << (r & 31));
      // Each thread copies one 16-byte column c of every (kProducerThreads / CH)-th row, for
      // Q, K and V: a warp covers whole 128-byte head rows, so every request is coalesced.
      const uint32_t stage = sb + OFF_STAGE + s * kStageBytes;
      constexpr int kRowsPerPass = kProducerThreads / CH;
      const int c = p % CH;
      const long long coff = static_cast<long long>(head) * HD + c * 8;
#pragma unroll 4
      for (int r = p / CH; r < kN; r += kRowsPerPass) {
        const int tk = tb.tok[r];
        const long long off = tk < 0 ? 0ll : static_cast<long long>(tk) * g.qkv_stride + coff;
        const uint32_t dst = stage + r * kRowBytes + ((c ^ (r & 7)) << 4);
        cp_async_16_zfill(dst, q + off, tk >= 0);
        cp_async_16_zfill(dst + kTileBytes, k + off, tk >= 0);
        cp_async_16_zfill(dst + 2 * kTileBytes, v + off, tk >= 0);
      }
      cp_async_commit();
      if (it > 0) {
        cp_async_wait_1();
        fence_proxy_async_smem();
        mbar_arrive(full_bar((it - 1) % kStages));
      }
    }
    cp_async_wait_0();
    fence_proxy_async_smem();
    if (!stopped && it > 0) mbar_arrive(full_bar((it - 1) % kStages));
  } else if (warp == 4) {
    // ------------------------------------------------------------------ MMA issuer
    // Issue order: S(t+1) goes out as soon as tile t+1 is loaded and S(t) has been read
    // out of TMEM, before PV(t); the softmax warps then find S(t+1) ready when they finish
    // tile t, and PV(t) runs underneath the softmax of tile t+1.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, kN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, HD, false, true);
    bool issued = false;
    auto issue_s = [&](int jt) -> bool {   // S(jt) = Q K^T of the tile in stage jt % kStages
      const int s = jt % kStages;
      if (!mbar_wait_bounded(full_bar(s), (jt / kStages) & 1, limit_ns)) return false;
      if (!mbar_wait_bounded(s_empty, (jt & 1) ^ 1, limit_ns)) return false;
      tc_fence_after();
      const uint32_t qa = sb + OFF_STAGE + s * kStageBytes, ka = qa + kTileBytes;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk)
        umma_bf16_ss(tmem + TM_S0, desc_kmajor_sw128(qa + kk * 32), desc_kmajor_sw128(ka + kk * 32), idesc_s, kk > 0);
      if (has_tail) {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_bf16_ss(tmem + TM_S1, desc_kmajor_sw128(qa + 128 * kRowBytes + kk * 32),
                       desc_kmajor_sw128(ka + kk * 32), idesc_s, kk > 0);
      }
      umma_commit(s_full);
      issued = true;
      return true;
    };
    auto issue_pv = [&](int jt) -> bool {  // O(jt) = P V of the tile in stage jt % kStages
      const int s = jt % kStages;
      if (!mbar_wait_bounded(p_full, jt & 1, limit_ns)) return false;
      if (!mbar_wait_bounded(o_empty, (jt & 1) ^ 1, limit_ns)) return false;
      tc_fence_after();
      const uint32_t va = sb + OFF_STAGE + s * kStageBytes + 2 * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < kN / 16; ++kk) {
        const uint64_t vd = desc_mnmajor_sw128(va + kk * 2048);
        const uint64_t pd0 = kk < 8 ? desc_kmajor_sw128(sb + (kk < 4 ? OFF_P0B0 : OFF_P0B1) + (kk & 3) * 32)
                                    : desc_kmajor_sw32(sb + OFF_P0B2);
        umma_bf16_ss(tmem + TM_O0, pd0, vd, idesc_o, kk > 0);
      }
      if (has_tail) {
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk) {
          const uint64_t vd = desc_mnmajor_sw128(va + kk * 2048);
          const uint64_t pd1 = kk < 8 ? desc_kmajor_sw128(sb + (kk < 4 ? OFF_P1B0 : OFF_P1B1) + (kk & 3) * 32)
                                      : desc_kmajor_sw32(sb + OFF_P1B2);
          umma_bf16_ss(tmem + TM_O1, pd1, vd, idesc_o, kk > 0);
        }
      }
      umma_commit(o_full);
      umma_commit(p_empty);
      umma_commit(empty_bar(s));
      return true;
    };
    int ok = 1;
    if (lane == 0 && static_cast<long long>(blockIdx.x) < num_tiles) ok = issue_s(0);
    int it = 0;
    for (long long tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
      if (lane == 0) {
        ok = !*abort_flag;
        if (ok && tile + gridDim.x < num_tiles) ok = issue_s(it + 1);
        if (ok) ok = issue_pv(it);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
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
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const float c = g.scale_log2;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const bool tail_warp = (warp == 0) && has_tail;
    int it = 0;
    // state of the previous tile, finished one iteration later
    bool have_prev = false;
    int prev_it = 0, prev_head = 0, prev_tok = -1, prev_tok_tail = -1;
    float prev_inv = 0.f, prev_inv_tail = 0.f;
    bool aborted = false;

    auto epilogue = [&](int pit, int head, int tok, int tok_tail, float inv, float inv_tail) -> bool {
      bool ok = mbar_wait_bounded(o_full, pit & 1, limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      tc_fence_after();
      float ov[HD], ov1[HD];
#pragma unroll
      for (int j = 0; j < HD / 16; ++j) tmem_ld16(tmem + lane_base + TM_O0 + 16 * j, ov + 16 * j);
      if (tail_warp) {
#pragma unroll
        for (int j = 0; j < HD / 16; ++j) tmem_ld16(tmem + lane_base + TM_O1 + 16 * j, ov1 + 16 * j);
      }
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < HD / 16; ++j) reg_fence16(ov + 16 * j);
      if (tail_warp) {
#pragma unroll
        for (int j = 0; j < HD / 16; ++j) reg_fence16(ov1 + 16 * j);
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      auto store_row = [&](const float* vals, float scl, int tk) {
        if (tk < 0) return;
        if constexpr (OUT_F32) {
          float* dst = static_cast<float*>(o) + static_cast<long long>(tk) * g.o_stride + head * HD;
#pragma unroll
          for (int j = 0; j < HD; j += 4)
            *reinterpret_cast<float4*>(dst + j) =
                make_float4(vals[j] * scl, vals[j + 1] * scl, vals[j + 2] * scl, vals[j + 3] * scl);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o) + static_cast<long long>(tk) * g.o_stride + head * HD;
#pragma unroll
          for (int j = 0; j < HD; j += 8) {
            uint4 u;
            u.x = pack_bf16x2(vals[j] * scl, vals[j + 1] * scl);
            u.y = pack_bf16x2(vals[j + 2] * scl, vals[j + 3] * scl);
            u.z = pack_bf16x2(vals[j + 4] * scl, vals[j + 5] * scl);
            u.w = pack_bf16x2(vals[j + 6] * scl, vals[j + 7] * scl);
            *reinterpret_cast<uint4*>(dst + j) = u;
          }
        }
      };
      store_row(ov, inv, tok);
      if (tail_warp && lane < 16) store_row(ov1, inv_tail, tok_tail);
      return true;
    };

    // Softmax of one S row held in registers: mask, row max, exp2, row sum (8 independent
    // accumulators each, so the reductions are not one long dependency chain).  The
    // probabilities stay in sv; returns 1 / rowsum.
    auto softmax_row = [&](float (&sv)[kN], const uint32_t (&mw)[kMaskWords], bool full_tile) -> float {
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = -INFINITY;
      if (full_tile) {
#pragma unroll
        for (int j = 0; j < kN; ++j) mx[j & 7] = fmaxf(mx[j & 7], sv[j]);
      } else {
#pragma unroll
        for (int j = 0; j < kN; ++j) {
          sv[j] = ((mw[j >> 5] >> (j & 31)) & 1u) ? sv[j] : -INFINITY;
          mx[j & 7] = fmaxf(mx[j & 7], sv[j]);
        }
      }
      float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      if (m == -INFINITY) m = 0.f;
      const float mc = m * c;
      float ls[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) ls[a] = 0.f;
#pragma unroll
      for (int j = 0; j < kN; ++j) {
        sv[j] = ex2(fmaf(sv[j], c, -mc));
        ls[j & 7] += sv[j];
      }
      const float l = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      return l > 0.f ? 1.f / l : 0.f;
    };
    // Round a probability row to bf16 and store it as row `row` of the P operand (keys
    // 0..63 and 64..127 in 128B-swizzled blocks, keys 128..143 in a 32B-swizzled block).
    auto store_p_row = [&](const float (&sv)[kN], int row, uint32_t pb0, uint32_t pb1, uint32_t pb2) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint32_t base = (b == 0 ? pb0 : pb1) + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int j0 = 64 * b + 8 * ch;
          asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(base + ((ch ^ (row & 7)) << 4)),
                       "r"(pack_bf16x2(sv[j0], sv[j0 + 1])), "r"(pack_bf16x2(sv[j0 + 2], sv[j0 + 3])),
                       "r"(pack_bf16x2(sv[j0 + 4], sv[j0 + 5])), "r"(pack_bf16x2(sv[j0 + 6], sv[j0 + 7]))
                       : "memory");
        }
      }
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int j0 = 128 + 8 * ch;
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(pb2 + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4)),
                     "r"(pack_bf16x2(sv[j0], sv[j0 + 1])), "r"(pack_bf16x2(sv[j0 + 2], sv[j0 + 3])),
                     "r"(pack_bf16x2(sv[j0 + 4], sv[j0 + 5])), "r"(pack_bf16x2(sv[j0 + 6], sv[j0 + 7]))
                     : "memory");
      }
    };

    for (long long tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) {
        aborted = true;
        break;
      }
      bool ok = mbar_wait_bounded(full_bar(s), ph, limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        aborted = true;
        break;
      }
      const long long win = tile / g.heads;
      const int head = static_cast<int>(tile - win * g.heads);
      const Table& tb = tables[s];
      const int tok = tb.tok[tid];
      uint32_t mw[kMaskWords], tw[kMaskWords];
      {
        const int lab = tb.lab[tid];
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) mw[w] = tb.mask[lab * kMaskWords + w];
      }
      int tok_tail = -1;
      if (tail_warp) {
        const int r = 128 + (lane & 15);
        tok_tail = lane < 16 ? tb.tok[r] : -1;
        const int lab = tb.lab[r];
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) tw[w] = tb.mask[lab * kMaskWords + w];
      }
      mbar_arrive(empty_bar(s));

      ok = mbar_wait_bounded(s_full, it & 1, limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float sv[kN];
#pragma unroll
      for (int j = 0; j < kN / 16; ++j) tmem_ld16(tmem + lane_base + TM_S0 + 16 * j, sv + 16 * j);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < kN / 16; ++j) reg_fence16(sv + 16 * j);
      if (!tail_warp) {
        tc_fence_before();
        mbar_arrive(s_empty);
      }
      const bool mfull = ((mw[0] & mw[1] & mw[2] & mw[3]) == 0xffffffffu) && ((mw[4] & 0xffffu) == 0xffffu);
      const bool full_tile = __all_sync(0xffffffffu, mfull);
      const float inv = softmax_row(sv, mw, full_tile);
      // P may only be overwritten once the previous tile's PV MMA has consumed it.
      ok = mbar_wait_bounded(p_empty, (it & 1) ^ 1, limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        aborted = true;
        break;
      }
      store_p_row(sv, tid, sb + OFF_P0B0, sb + OFF_P0B1, sb + OFF_P0B2);
      float inv_tail = 0.f;
      if (tail_warp) {
#pragma unroll
        for (int j = 0; j < kN / 16; ++j) tmem_ld16(tmem + lane_base + TM_S1 + 16 * j, sv + 16 * j);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kN / 16; ++j) reg_fence16(sv + 16 * j);
        tc_fence_before();
        mbar_arrive(s_empty);
        const bool tfull = ((tw[0] & tw[1] & tw[2] & tw[3]) == 0xffffffffu) && ((tw[4] & 0xffffu) == 0xffffu);
        const bool tfull_w = __all_sync(0xffffffffu, tfull || lane >= 16);
        inv_tail = softmax_row(sv, tw, tfull_w);
        if (lane < 16) store_p_row(sv, lane, sb + OFF_P1B0, sb + OFF_P1B1, sb + OFF_P1B2);
      }
      fence_proxy_async_smem();
      mbar_arrive(p_full);
      if (have_prev) {
        if (!epilogue(prev_it, prev_head, prev_tok, prev_tok_tail, prev_inv, prev_inv_tail)) {
          aborted = true;
          have_prev = false;
          break;
        }
      }
      have_prev = true;
      prev_it = it;
      prev_head = head;
      prev_tok = tok;
      prev_tok_tail = tok_tail;
      prev_inv = inv;
      prev_inv_tail = inv_tail;
    }
    if (have_prev && !aborted) {
      if (!epilogue(prev_it, prev_head, prev_tok, prev_tok_tail, prev_inv, prev_inv_tail)) aborted = true;
    }
    if (aborted) {
      if (lane == 0) record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, kTmemCols);
}

template <int HD, bool OUT_F32>
cudaError_t launch_t(const WinGeom& g, const void* q, const void* k, const void* v, void* o, int* err,
                     long long limit_ns, int num_sms, cudaStream_t st) {
  auto kern = window_attn_tc_kernel<HD, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  const long long tiles = g.windows * g.heads;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, kThreads, kSmemAlloc, st>>>(g, static_cast<const __nv_bfloat16*>(q),
                                           static_cast<const __nv_bfloat16*>(k),
                                           static_cast<const __nv_bfloat16*>(v), o, err,
                                           static_cast<unsigned long long>(limit_ns < 0 ? 0 : limit_ns));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn_tc(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                  bool out_f32, int* err, long long spin_limit, int num_sms, cudaStream_t stream) {
  if (g.head_dim == 64)
    return out_f32 ? launch_t<64, true>(g, q, k, v, o, err, spin_limit, num_sms, stream)
                   : launch_t<64, false>(g, q, k, v, o, err, spin_limit, num_sms, stream);
  return out_f32 ? launch_t<32, true>(g, q, k, v, o, err, spin_limit, num_sms, stream)
                 : launch_t<32, false>(g, q, k, v, o, err, spin_limit, num_sms, stream);
}

}  // namespace s3w
