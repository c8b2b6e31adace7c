// Shifted-window attention for windows larger than one 144-slot tile (N > 144): the
// multi-block streaming path.  Each window is cut into blocks of consecutive whole (t, h)
// rows (a block may span T-slabs), at most 128 slots each.  A unit of work is one (window,
// head, query block); the
// window's K/V blocks stream past it through a TMA ring, and the softmax is carried across
// key blocks online (running row max, rescaled row sum and output), so any N fits.
//
// Method: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
// section "CuTe DSL window attention" (per window and head S = scale * Q K^T, the shift
// mask, FP32 softmax, O = softmax(S) V, BF16 operands with FP32 accumulation; where a window
// outgrows the single-stage path, K/V tiles are streamed with online-softmax rescaling).
// Shift, pad, partition and merge are folded into the gather and scatter as in the
// single-tile kernel (section "Kernel fusion for backbone memory traffic").
//
// Per CTA (persistent, one per SM), 11 warps:
//   softmax warps 0..7  thread (row = 32 (w % 4) + lane of the query block, key half w / 4):
//                       per key block, 64 logits from TMEM, the key mask of the query's
//                       region combination, the row max across both halves (shared memory),
//                       the online update, and P (bf16) written back over the thread's own
//                       logit columns in TMEM; then the previous block's P V is folded into
//                       the running output (registers).  After the last key block the row
//                       is divided by its sum and stored to the query's grid position.
//   MMA warp 8          S(j) = Q K(j)^T (M = 128, N = key slots rounded up to 16) into one
//                       of two TMEM buffers, then O(j) = P(j) [V(j) | 1] with P read from
//                       TMEM (the A operand of the TS form) and V plus a block of ones from
//                       shared memory: O's columns 64.. are the row sums of the bf16 P.
//   TMA warp 9          the unit's Q block (two buffers) and every K/V block through a
//                       four-stage ring: per run of rows inside one T-slab and one side of
//                       the H seam, boxes of 2^k rows; one row at a time (cut in two) where
//                       the window wraps around the W seam.  Padded coordinates read as zero.
//   table warp 10       per K/V block, the visible keys for each of the 8 combinations of a
//                       query's wrapped-around sides.
// Every wait is bounded; a timeout unwinds the CTA (error word set, copies drained, TMEM
// freed).
#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_common.cuh"
#include "s3w_internal.h"
#include "sm100_ptx.cuh"

namespace s3w {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kBlk = 128;                     // slots per block at most (query rows, keys)
constexpr int kBlkBytes = kBlk * kRowBytes;   // one tensor's block: 16 KB
constexpr int kStagesS = 4;
constexpr int kThreadsS = 352;
constexpr int kMmaWarpS = 8, kTmaWarpS = 9, kTableWarpS = 10;

// TMEM columns: S of two key blocks (by block parity), 128 columns each.  P is written back
// over the first 32 columns of each key half's 64 logit columns: keys 16k .. 16k + 15 are at
// column 64 (k / 4) + 8 (k % 4) (two bf16 per column).  O (64 value columns, then 16 copies
// of the row sum) after them.
constexpr uint32_t TS_S = 0, TS_O = 256, kSumCol = 64;

// Box shapes of the tensor maps: 2^k (t, h) rows of win_w tokens (k = 0..7; a run of rows
// is loaded as its binary decomposition), and a row cut at the W seam (win_w - shift_w
// tokens, then shift_w).
constexpr int kRowShapes = 8;
enum : int { kBoxW1 = kRowShapes, kBoxW2 = kRowShapes + 1, kBoxShapesS = kRowShapes + 2 };
struct StreamMaps {
  CUtensorMap m[3][kBoxShapesS];   // [tensor q/k/v][box shape]
};

// How a window is cut into blocks: its (t, h) rows, numbered R = t win_h + h, in runs of
// `nr` consecutive rows (the last may be shorter), at most 128 slots each; a block may span
// two or more T-slabs.
struct StreamPlan {
  int nr;        // rows per block
  int nblk;      // blocks per window (= query blocks = key blocks)
  long long units;   // windows * heads * nblk
};

// Per K/V stage: bit i of mask[c][w] = key 32 w + i of the block is visible to a query whose
// wrapped-around sides are c (bit a: axis a).
struct KeyTable {
  uint32_t mask[8][4];
};

struct SmemS {
  static constexpr int OFF_Q = 0;                                    // Q blocks, by unit parity
  static constexpr int OFF_KV = OFF_Q + 2 * kBlkBytes;              // stages of (K, V)
  static constexpr int OFF_ONES = OFF_KV + kStagesS * 2 * kBlkBytes;   // 16 key rows of bf16 ones
  static constexpr int OFF_TAB = OFF_ONES + 16 * kRowBytes;
  static constexpr int OFF_BARS = OFF_TAB + kStagesS * static_cast<int>(sizeof(KeyTable));
  // q_full[2], q_free[2], kv_full[S], kv_empty[S], tab_full[S], s_full[2], s_free[2],
  // p_full[2], o_full, o_empty, row max written[2 parity][2 half], drain
  static constexpr int kNumBars = 4 + 3 * kStagesS + 6 + 2 + 4 + 1;
  static constexpr int OFF_XCHG = OFF_BARS + kNumBars * 8;            // float [2 parity][2 half][128]
  static constexpr int OFF_MISC = OFF_XCHG + 2 * 2 * 128 * 4;         // tmem address, abort flag
  static constexpr int kBytes = OFF_MISC + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
  static_assert(OFF_BARS % 8 == 0, "mbarrier alignment");
};

// Rows of block b: window rows [r0, r0 + nr) (row R = t win_h + h).
struct BlockRows {
  int r0, nr;
};
__device__ __forceinline__ BlockRows block_rows(const WinGeom& g, const StreamPlan& sp, int b) {
  BlockRows br;
  br.r0 = b * sp.nr;
  br.nr = min(sp.nr, g.wt * g.wh - br.r0);
  return br;
}

// Loads block b of tensor `tsr` of the tile into `dst` (slot i of the block at row i) and
// completes its bytes on `bar`.  Rows of one T-slab on one side of the H seam form a run,
// loaded as boxes of 2^k rows (its binary decomposition); where the window wraps around the
// W seam, every row is two boxes.
__device__ __forceinline__ void load_block(const WinGeom& g, const StreamPlan& sp, const StreamMaps& maps, int tsr,
                                           const TileCoord& tc, int b, uint32_t dst, uint32_t bar) {
  const BlockRows br = block_rows(g, sp, b);
  const int c0 = tc.head * g.head_dim;
  const bool wrap_w = tc.bw + g.ww > g.Pw;
  const int n1h = g.Ph - tc.bh;   // window rows (h) before the H seam
  const int n1w = g.Pw - tc.bw;   // window columns before the W seam
  const uint32_t row_bytes = static_cast<uint32_t>(g.ww * kRowBytes);
  int rt = br.r0 / g.wh, rh = br.r0 - rt * g.wh;
  int done = 0;
#pragma unroll 1
  while (done < br.nr) {
    int t = tc.bt + rt;
    t -= t >= g.Pt ? g.Pt : 0;
    // the run: rows of this slab, up to the H seam or the slab's end
    const int lim = rh < n1h ? min(g.wh, n1h) : g.wh;
    const int n = min(br.nr - done, lim - rh);
    int h = tc.bh + rh;
    h -= h >= g.Ph ? g.Ph : 0;
    uint32_t d = dst + static_cast<uint32_t>(done) * row_bytes;
    if (!wrap_w) {
#pragma unroll 1
      for (int k = kRowShapes - 1; k >= 0; --k) {
        if (!((n >> k) & 1)) continue;
        tma_load_5d(d, &maps.m[tsr][k], c0, tc.bw, h, t, tc.bsmp, bar);
        d += static_cast<uint32_t>(1 << k) * row_bytes;
        h += 1 << k;
      }
    } else {
#pragma unroll 1
      for (int r = 0; r < n; ++r, d += row_bytes, ++h) {
        tma_load_5d(d, &maps.m[tsr][kBoxW1], c0, tc.bw, h, t, tc.bsmp, bar);
        tma_load_5d(d + static_cast<uint32_t>(n1w * kRowBytes), &maps.m[tsr][kBoxW2], c0, 0, h, t, tc.bsmp, bar);
      }
    }
    done += n;
    rh += n;
    if (rh == g.wh) {
      rh = 0;
      ++rt;
    }
  }
}

// The grid token of slot i of block b (-1 if padded) and its wrapped-around sides.
__device__ __forceinline__ int block_slot(const WinGeom& g, const TileCoord& tc, const BlockRows& br, int i,
                                          uint32_t* sides) {
  const int row = br.r0 + i / g.ww, rw = i - (i / g.ww) * g.ww;
  const int rt = row / g.wh, rh = row - rt * g.wh;
  *sides = (rt >= g.wt - g.st ? 1u : 0u) | (rh >= g.wh - g.sh ? 2u : 0u) | (rw >= g.ww - g.sw ? 4u : 0u);
  int t = tc.bt + rt, h = tc.bh + rh, w = tc.bw + rw;
  t -= t >= g.Pt ? g.Pt : 0;
  h -= h >= g.Ph ? g.Ph : 0;
  w -= w >= g.Pw ? g.Pw : 0;
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return ((tc.bsmp * g.T + t) * g.H + h) * g.W + w;
}

// Word w (bits 32 w .. 32 w + 31) of the 128-bit set of indices in [lo, hi).
__device__ __forceinline__ uint32_t range_word(int lo, int hi, int w) {
  const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 32);
  if (b <= a) return 0u;
  return (b - a == 32) ? 0xffffffffu : (((1u << (b - a)) - 1u) << a);
}

// 32 bits of the 128-bit set (c0, c1, c2, c3) starting at bit a (0 <= a < 128; zeros past
// the end), with register selects instead of an indexed array.
__device__ __forceinline__ uint32_t bits_at(const uint32_t (&c)[4], int a) {
  const int w = a >> 5;
  const uint32_t x = w == 0 ? c[0] : (w == 1 ? c[1] : (w == 2 ? c[2] : c[3]));
  const uint32_t y = w == 0 ? c[1] : (w == 1 ? c[2] : (w == 2 ? c[3] : 0u));
  return __funnelshift_r(x, y, static_cast<uint32_t>(a & 31));
}

// Offsets r in [0, w) of a window axis whose coordinate (base + r, wrapped at P) lies inside
// the unpadded extent D: [0, min(P - base, D - base)) and, past the seam, [P - base,
// min(w, P - base + D)).
struct RealRange {
  int a1, b1, a2, b2;
};
__device__ __forceinline__ RealRange real_range(int base, int w, int P, int D) {
  RealRange r;
  const int n1 = P - base;
  r.a1 = 0;
  r.b1 = min(min(n1, w), D - base);
  r.a2 = n1;
  r.b2 = min(w, n1 + D);
  return r;
}
__device__ __forceinline__ bool in_real(const RealRange& r, int x) {
  return (x >= r.a1 && x < r.b1) || (x >= r.a2 && x < r.b2);
}

// O (+)= P [V | 1] over `ksteps` (1..8) K steps of 16 keys, one asm block: A (P, bf16) from
// TMEM at column 64 (k / 4) + 8 (k % 4) of the S buffer, B (V, MN-major) from shared memory
// moving 2048 bytes per step while its leading byte offset (the ones block behind it) moves
// back as much (-8388480 = 2048 / 16 - (2048 / 16 << 16) in descriptor units).  Steps past
// `ksteps` are predicated off.  Executed by the whole warp; only `leader` issues.
#define S3W_PV_STEP_(K, AOFF)                                                                     \
  "add.s64 b, b, -8388480;\n\tadd.u32 a, %1, " AOFF ";\n\tsetp.gt.and.s32 p, %5, " K ", q;\n\t" \
  "@p tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, t;\n\t"
__device__ __forceinline__ void umma_pv_ts(uint32_t d_tmem, uint32_t p_tmem, uint64_t v0, int ksteps, uint32_t idesc,
                                           uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred q, p, f, t;\n\t.reg .b64 b;\n\t.reg .b32 a;\n\t"
      "setp.ne.b32 q, %4, 0;\n\tsetp.ne.b32 f, %4, %4;\n\tsetp.eq.b32 t, %4, %4;\n\t"
      "mov.b64 b, %2;\n\t@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b, %3, f;\n\t"
      S3W_PV_STEP_("1", "8") S3W_PV_STEP_("2", "16") S3W_PV_STEP_("3", "24") S3W_PV_STEP_("4", "64")
      S3W_PV_STEP_("5", "72") S3W_PV_STEP_("6", "80") S3W_PV_STEP_("7", "88") "}" ::"r"(d_tmem),
      "r"(p_tmem), "l"(v0), "r"(idesc), "r"(leader), "r"(ksteps)
      : "memory");
}
#undef S3W_PV_STEP_

__device__ __forceinline__ void tmem_wait_st_s() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 8 consecutive columns, registers -> TMEM (thread t: lane base + t).
__device__ __forceinline__ void tmem_st8_s(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

template <int HD, bool OUT_F32>
__global__ void __launch_bounds__(kThreadsS, 1)
window_attn_stream_kernel(const __grid_constant__ WinGeom g, const __grid_constant__ StreamMaps maps,
                          const StreamPlan sp, void* __restrict__ o, int* __restrict__ err,
                          unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  KeyTable* tabs = reinterpret_cast<KeyTable*>(sm + SmemS::OFF_TAB);
  const uint32_t bar0 = sb + SmemS::OFF_BARS;
  auto q_full = [&](int b) { return bar0 + 8u * b; };
  auto q_free = [&](int b) { return bar0 + 8u * (2 + b); };
  auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + kStagesS + s); };
  auto tab_full = [&](int s) { return bar0 + 8u * (4 + 2 * kStagesS + s); };
  constexpr int kB = 4 + 3 * kStagesS;
  auto s_full = [&](int b) { return bar0 + 8u * (kB + b); };
  auto s_free = [&](int b) { return bar0 + 8u * (kB + 2 + b); };
  auto p_full = [&](int b) { return bar0 + 8u * (kB + 4 + b); };
  const uint32_t o_full = bar0 + 8u * (kB + 6);
  const uint32_t o_empty = bar0 + 8u * (kB + 7);
  auto xmax_bar = [&](int par, int h) { return bar0 + 8u * (kB + 8 + 2 * par + h); };
  const uint32_t drain_bar = bar0 + 8u * (kB + 12);
  float* xmax = reinterpret_cast<float*>(sm + SmemS::OFF_XCHG);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + SmemS::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SmemS::OFF_MISC + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long my_units =
      static_cast<long long>(blockIdx.x) < sp.units ? (sp.units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto unit_of = [&](long long ui) { return blockIdx.x + ui * gridDim.x; };

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_free(b), 1);
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 1);
      mbar_init(p_full(b), 256);
    }
    for (int s = 0; s < kStagesS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1 + 256);   // PV commit + every softmax thread (its table read)
      mbar_init(tab_full(s), 32);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, 256);
    for (int par = 0; par < 2; ++par)
      for (int h = 0; h < 2; ++h) mbar_init(xmax_bar(par, h), 128);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // Rows of a block beyond its slots are never loaded: start every buffer at zero (finite),
  // and fill the ones block (bf16 1.0 = 0x3f80).
  for (int i = tid; i < SmemS::OFF_ONES / 16; i += kThreadsS)
    *reinterpret_cast<uint4*>(sm + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < 16 * kRowBytes / 16; i += kThreadsS)
    *reinterpret_cast<uint4*>(sm + SmemS::OFF_ONES + 16 * i) =
        make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
  fence_proxy_async_smem();
  if (warp == kMmaWarpS) {
    tmem_alloc(sb + SmemS::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t qbuf0 = sb + SmemS::OFF_Q;
  auto kbuf = [&](int s) { return sb + SmemS::OFF_KV + static_cast<uint32_t>(s * 2 * kBlkBytes); };

  if (warp == kTmaWarpS) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
#pragma unroll
      for (int a = 0; a < 3; ++a)
#pragma unroll
        for (int b = 0; b < kBoxShapesS; ++b) prefetch_tmap(&maps.m[a][b]);
      long long j = 0, nq = 0;   // K/V blocks and Q blocks issued
      bool ok = true;
      for (long long ui = 0; ok && ui < my_units; ++ui) {
        const long long u = unit_of(ui);
        const long long tile = u / sp.nblk;
        const int qb = static_cast<int>(u - tile * sp.nblk);
        const TileCoord tc = tile_coord(g, tile);
        const int qp = static_cast<int>(ui & 1);
        if (*abort_flag || !mbar_wait_bounded(q_free(qp), static_cast<uint32_t>(((ui >> 1) & 1) ^ 1), limit_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full(qp), static_cast<uint32_t>(block_rows(g, sp, qb).nr * g.ww * kRowBytes));
        load_block(g, sp, maps, 0, tc, qb, qbuf0 + static_cast<uint32_t>(qp * kBlkBytes), q_full(qp));
        ++nq;
        for (int kb = 0; kb < sp.nblk; ++kb, ++j) {
          const int s = static_cast<int>(j % kStagesS);
          if (*abort_flag ||
              !mbar_wait_bounded(kv_empty(s), static_cast<uint32_t>(((j / kStagesS) & 1) ^ 1), limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t bytes = static_cast<uint32_t>(2 * block_rows(g, sp, kb).nr * g.ww * kRowBytes);
          mbar_arrive_expect_tx(kv_full(s), bytes);
          load_block(g, sp, maps, 1, tc, kb, kbuf(s), kv_full(s));
          load_block(g, sp, maps, 2, tc, kb, kbuf(s) + kBlkBytes, kv_full(s));
        }
      }
      if (!ok) {
        record_error(err, kStatusTimeout);
        *abort_flag = 1;
      }
      // Every load issued must land before the CTA exits (bounded, independent of the test
      // limit): the last stages and Q buffers issued.
      for (long long jj = j > kStagesS ? j - kStagesS : 0; jj < j; ++jj)
        if (!mbar_wait_bounded(kv_full(static_cast<int>(jj % kStagesS)), static_cast<uint32_t>((jj / kStagesS) & 1),
                               2000000000ull))
          record_error(err, kStatusTimeout);
      for (long long qi = nq > 2 ? nq - 2 : 0; qi < nq; ++qi)
        if (!mbar_wait_bounded(q_full(static_cast<int>(qi & 1)), static_cast<uint32_t>((qi >> 1) & 1), 2000000000ull))
          record_error(err, kStatusTimeout);
    }
  } else if (warp == kTableWarpS) {
    // ------------------------------------------------------------------ key tables
    // Lane L fills word L % 4 (keys 32 (L % 4) ..) of combination L / 4.  The visibility of
    // a key factors by axis: its T-slab (per block), its (t, h) row and its column.  Per
    // window the visible columns of the lane's combination are a 128-bit set built from index
    // intervals; a block's word then walks its keys row by row without divisions.
    const uint32_t combo = static_cast<uint32_t>(lane) >> 2;
    const int word = lane & 3;
    long long j = 0;
    bool ok = true;
    for (long long ui = 0; ok && ui < my_units; ++ui) {
      const long long u = unit_of(ui);
      const long long tile = u / sp.nblk;
      const TileCoord tc = tile_coord(g, tile);
      // sides that split the window's regions: axes along which it is the last window of
      // a shifted axis
      const bool last_t = tc.itw == g.nwt - 1 && g.st > 0, last_h = tc.ih == g.nwh - 1 && g.sh > 0,
                 last_w = tc.iw == g.nww - 1 && g.sw > 0;
      const RealRange rt_r = real_range(tc.bt, g.wt, g.Pt, g.T);
      const RealRange rh_r = real_range(tc.bh, g.wh, g.Ph, g.H);
      const RealRange rw_r = real_range(tc.bw, g.ww, g.Pw, g.W);
      uint32_t colok[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t real = range_word(rw_r.a1, rw_r.b1, q4) | range_word(rw_r.a2, rw_r.b2, q4);
        if (last_w) {
          const uint32_t side = range_word(g.ww - g.sw, g.ww, q4);
          real &= (combo & 4u) ? side : ~side;
        }
        colok[q4] = real;
      }
      for (int kb = 0; kb < sp.nblk; ++kb, ++j) {
        const int s = static_cast<int>(j % kStagesS);
        if (__any_sync(0xffffffffu, *abort_flag != 0) ||
            !__all_sync(0xffffffffu, mbar_wait_bounded(kv_empty(s), static_cast<uint32_t>(((j / kStagesS) & 1) ^ 1),
                                                       limit_ns))) {
          ok = false;
          break;
        }
        const BlockRows br = block_rows(g, sp, kb);
        const int nb = br.nr * g.ww;
        auto row_ok = [&](int row) {   // row of the block -> its (t, h) visible for the combination
          const int rr = br.r0 + row;
          const int rt = rr / g.wh, rh = rr - rt * g.wh;
          return row < br.nr && in_real(rt_r, rt) && (!last_t || (rt >= g.wt - g.st) == ((combo & 1u) != 0)) &&
                 in_real(rh_r, rh) && (!last_h || (rh >= g.wh - g.sh) == ((combo & 2u) != 0));
        };
        // the word's keys [i0, i1) are key = row * win_w + col: per (t, h) row overlapping
        // them, that row's visible columns shifted into place
        uint32_t bits = 0;
        const int i0 = 32 * word, i1 = min(i0 + 32, nb);
        if (i0 < i1) {
          int row = i0 / g.ww;
#pragma unroll 1
          for (int base = row * g.ww; base < i1; base += g.ww, ++row) {
            if (!row_ok(row)) continue;
            const int lo = max(base, i0), hi = min(base + g.ww, i1);
            const int len = hi - lo;
            const uint32_t seg = bits_at(colok, lo - base) & (len >= 32 ? 0xffffffffu : ((1u << len) - 1u));
            bits |= seg << (lo - i0);
          }
        }
        tabs[s].mask[combo][word] = bits;
        __syncwarp();
        mbar_arrive(tab_full(s));
      }
    }
    if (!ok && lane == 0) {
      record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  } else if (warp == kMmaWarpS) {
    // ------------------------------------------------------------------ MMA issuer
    // Block j of the CTA (unit j / nblk, key block j % nblk): S(j) into buffer j % 2 once
    // PV(j - 2) has freed it, then PV(j - 1); the order S(0); S(1), PV(0); S(2), PV(1); ...
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, kSumCol + 16, false, true);
    const uint32_t leader = lane == 0 ? 1u : 0u;
    bool issued = false;
    auto ksteps_of = [&](int kb) { return (block_rows(g, sp, kb).nr * g.ww + 15) >> 4; };
    auto issue_s = [&](long long jj) -> bool {
      const long long ui = jj / sp.nblk;
      const int kb = static_cast<int>(jj - ui * sp.nblk);
      const int s = static_cast<int>(jj % kStagesS), buf = static_cast<int>(jj & 1), qp = static_cast<int>(ui & 1);
      if (kb == 0 &&
          !__all_sync(0xffffffffu, mbar_wait_bounded(q_full(qp), static_cast<uint32_t>((ui >> 1) & 1), limit_ns)))
        return false;
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(kv_full(s), static_cast<uint32_t>((jj / kStagesS) & 1), limit_ns)))
        return false;
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(s_free(buf), static_cast<uint32_t>(((jj >> 1) & 1) ^ 1), limit_ns)))
        return false;
      tc_fence_after();
      const int nkeys = ksteps_of(kb) * 16;
      const uint64_t qd = smem_desc(qbuf0 + static_cast<uint32_t>(qp * kBlkBytes), 16, 1024, kSwizzle128B);
      const uint64_t kd = smem_desc(kbuf(s), 16, 1024, kSwizzle128B);
      umma_chain_qk<HD / 16>(tmem + TS_S + 128u * buf, qd, kd, idesc_bf16_f32(128, nkeys, false, false), leader);
      umma_commit_leader(s_full(buf), leader);
      if (kb == sp.nblk - 1) umma_commit_leader(q_free(qp), leader);
      issued = true;
      return true;
    };
    auto issue_pv = [&](long long jj) -> bool {
      const long long ui = jj / sp.nblk;
      const int kb = static_cast<int>(jj - ui * sp.nblk);
      const int s = static_cast<int>(jj % kStagesS), buf = static_cast<int>(jj & 1);
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(p_full(buf), static_cast<uint32_t>((jj >> 1) & 1), limit_ns)))
        return false;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_empty, static_cast<uint32_t>((jj & 1) ^ 1), limit_ns)))
        return false;
      tc_fence_after();
      const uint32_t vaddr = kbuf(s) + kBlkBytes;
      const uint32_t ones = sb + SmemS::OFF_ONES;
      const uint64_t vd = smem_desc(vaddr, ones - vaddr, 1024, kSwizzle128B);
      umma_pv_ts(tmem + TS_O, tmem + TS_S + 128u * buf, vd, ksteps_of(kb), idesc_o, leader);
      umma_commit_leader(o_full, leader);
      umma_commit_leader(kv_empty(s), leader);
      umma_commit_leader(s_free(buf), leader);
      return true;
    };
    // Failure injection (tests): wait on the drain barrier, which nothing signals before the
    // loop below has run, so the bounded wait expires and the CTA takes the timeout path.
    bool ok = !g.test_stall || __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, limit_ns));
    const long long nblocks = my_units * sp.nblk;
    for (long long jj = 0; ok && jj <= nblocks; ++jj) {
      ok = !__any_sync(0xffffffffu, *abort_flag != 0);
      if (ok && jj < nblocks) ok = issue_s(jj);
      if (ok && jj > 0) ok = issue_pv(jj - 1);
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
  } else {
    // ------------------------------------------------------------------ softmax + output
    const float c = g.scale_log2;
    const int half = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    long long j = 0;
    bool aborted = false;
    auto selb = [](uint32_t w, int e, float x) { return ((w >> e) & 1u) ? x : -INFINITY; };
    for (long long ui = 0; ui < my_units && !aborted; ++ui) {
      const long long u = unit_of(ui);
      const long long tile = u / sp.nblk;
      const int qb = static_cast<int>(u - tile * sp.nblk);
      const TileCoord tc = tile_coord(g, tile);
      const BlockRows qr = block_rows(g, sp, qb);
      uint32_t combo = 0;
      const int tok = row < qr.nr * g.ww ? block_slot(g, tc, qr, row, &combo) : -1;
      float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
      float acc[HD / 2];
#pragma unroll
      for (int e = 0; e < HD / 2; ++e) acc[e] = 0.f;
      // O(jj) into the running output, scaled by alpha.
      auto fold = [&](long long jj, float alpha) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(o_full, static_cast<uint32_t>(jj & 1), limit_ns))) return false;
        tc_fence_after();
        float ov[HD / 2], lb;
#pragma unroll
        for (int mm = 0; mm < HD / 32; ++mm) tmem_ld16(tmem + lane_base + TS_O + 32 * mm + 16 * half, ov + 16 * mm);
        tmem_ld1(tmem + lane_base + TS_O + kSumCol, &lb);
        tmem_wait_ld();
#pragma unroll
        for (int mm = 0; mm < HD / 32; ++mm) reg_fence16(ov + 16 * mm);
        reg_fence1(&lb);
        tc_fence_before();
        mbar_arrive(o_empty);
#pragma unroll
        for (int e = 0; e < HD / 2; ++e) acc[e] = fmaf(acc[e], alpha, ov[e]);
        l = fmaf(l, alpha, lb);
        return true;
      };
      for (int kb = 0; kb < sp.nblk; ++kb, ++j) {
        const int s = static_cast<int>(j % kStagesS), buf = static_cast<int>(j & 1), par = buf;
        if (__any_sync(0xffffffffu, *abort_flag != 0) ||
            !__all_sync(0xffffffffu,
                        mbar_wait_bounded(tab_full(s), static_cast<uint32_t>((j / kStagesS) & 1), limit_ns))) {
          aborted = true;
          break;
        }
        const uint32_t mw0 = tabs[s].mask[combo][2 * half], mw1 = tabs[s].mask[combo][2 * half + 1];
        mbar_arrive(kv_empty(s));
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(s_full(buf), static_cast<uint32_t>((j >> 1) & 1), limit_ns))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t sbase = tmem + lane_base + TS_S + 128u * buf + 64u * half;
        // the block's key columns (slots rounded up to 16) of this thread's half, in groups
        // of 8; the rest are never computed by the S MMA nor read by the PV MMA
        const int ng = min(max((((block_rows(g, sp, kb).nr * g.ww + 15) & ~15) - 64 * half) >> 3, 0), 8);
        // columns past the block hold stale values: their mask bits are 0
        float x[64];
#pragma unroll
        for (int k = 0; k < 8; ++k) tmem_ld8(sbase + 8 * k, x + 8 * k);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) reg_fence8(x + 8 * k);
        if (__any_sync(0xffffffffu, (mw0 & mw1) != 0xffffffffu)) {   // some key of the warp hidden
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            x[e] = selb(mw0, e, x[e]);
            x[32 + e] = selb(mw1, e, x[32 + e]);
          }
        }
        float a = -INFINITY, b = -INFINITY;
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          a = max3(a, x[e], x[e + 1]);
          b = max3(b, x[e + 2], x[e + 3]);
        }
        const float mh = fmaxf(a, b);
        xmax[(par * 2 + half) * 128 + row] = mh;
        mbar_arrive(xmax_bar(par, half));
        if (!__all_sync(0xffffffffu,
                        mbar_wait_bounded(xmax_bar(par, half ^ 1), static_cast<uint32_t>((j >> 1) & 1), limit_ns))) {
          aborted = true;
          break;
        }
        const float mb = fmaxf(mh, xmax[(par * 2 + (half ^ 1)) * 128 + row]);
        // online update: the new running max, the factor for what was accumulated so far
        const float m_new = fmaxf(m, mb);
        float alpha, mu;
        if (m_new == -INFINITY) {   // no visible key so far: P = 0, nothing to rescale
          alpha = 1.f;
          mu = 0.f;
        } else {
          alpha = ex2((m - m_new) * c);
          mu = m_new;
        }
        m = m_new;
        // P = exp2(c (x - m)) as bf16 pairs over the thread's first 32 logit columns
        const float2 cc = make_float2(c, c), nm = make_float2(-mu * c, -mu * c);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (2 * k >= ng) break;   // keys 16k .. of the half are past the block's columns
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 y = fma2(make_float2(x[16 * k + 2 * e], x[16 * k + 2 * e + 1]), cc, nm);
            pk[e] = pack_bf16x2_int(ex2(y.x), ex2(y.y));
          }
          tmem_st8_s(sbase + 8 * k, pk);
        }
        tmem_wait_st_s();
        tc_fence_before();
        mbar_arrive(p_full(buf));
        if (kb > 0 && !fold(j - 1, alpha_prev)) {
          aborted = true;
          break;
        }
        alpha_prev = alpha;
      }
      if (aborted) break;
      if (!fold(j - 1, alpha_prev)) {   // the unit's last key block
        aborted = true;
        break;
      }
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      store_o_row<HD, OUT_F32>(o, g.o_stride, g.o_rows_32b != 0, tok, tc.head, half, lane, acc, inv);
    }
    if (aborted) {
      if (lane == 0) record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarpS) tmem_dealloc(tmem, 512);
}

// Block plan: as few blocks as fit 128 slots each, the window's rows spread evenly.
StreamPlan make_plan(const WinGeom& g) {
  StreamPlan sp;
  const int rows = g.wt * g.wh;
  const int per_block = kBlk / g.ww;                  // rows that fit one block (win_w <= 128)
  sp.nblk = (rows + per_block - 1) / per_block;
  sp.nr = (rows + sp.nblk - 1) / sp.nblk;
  sp.nblk = (rows + sp.nr - 1) / sp.nr;
  sp.units = g.windows * g.heads * sp.nblk;
  return sp;
}

cudaError_t make_stream_maps(const WinGeom& g, const void* const ptrs[3], StreamMaps* maps) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t C = static_cast<cuuint64_t>(g.heads) * g.head_dim;
  const cuuint64_t dims[5] = {C, static_cast<cuuint64_t>(g.W), static_cast<cuuint64_t>(g.H),
                              static_cast<cuuint64_t>(g.T), static_cast<cuuint64_t>(g.B)};
  const cuuint64_t row = static_cast<cuuint64_t>(g.qkv_stride) * 2;
  const cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
  const cuuint32_t ww = static_cast<cuuint32_t>(g.ww), sw = static_cast<cuuint32_t>(g.sw);
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  for (int t = 0; t < 3; ++t)
    for (int b = 0; b < kBoxShapesS; ++b) {
      // 2^b rows of win_w tokens (a shape taller than any run of 128 slots is never used and
      // is encoded one row high); a seam shape of an unshifted axis is never used either
      cuuint32_t bw = ww, bh = 1;
      if (b < kRowShapes) {
        if ((static_cast<cuuint32_t>(1) << b) * ww <= static_cast<cuuint32_t>(kBlk)) bh = 1u << b;
      } else if (b == kBoxW1) {
        bw = sw > 0 ? ww - sw : ww;
      } else {
        bw = sw > 0 ? sw : ww;
      }
      const cuuint32_t box[5] = {static_cast<cuuint32_t>(kRowBytes / 2), bw, bh, 1, 1};
      CUresult r = enc(&maps->m[t][b], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptrs[t]), dims, strides,
                       box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
  return cudaSuccess;
}

template <int HD, bool OUT_F32>
cudaError_t launch_s(const WinGeom& g, const StreamMaps& maps, const StreamPlan& sp, void* o, int* err,
                     long long limit_ns, int num_sms, cudaStream_t st) {
  auto kern = window_attn_stream_kernel<HD, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemS::kAlloc);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(sp.units < num_sms ? sp.units : num_sms);
  kern<<<grid, kThreadsS, SmemS::kAlloc, st>>>(g, maps, sp, o, err,
                                                static_cast<unsigned long long>(limit_ns < 0 ? 0 : limit_ns));
  return cudaGetLastError();
}

}  // namespace

long long window_attn_stream_units(const WinGeom& g) { return make_plan(g).units; }

cudaError_t launch_window_attn_stream(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                      bool out_f32, int* err, long long spin_limit, int num_sms, cudaStream_t stream) {
  const StreamPlan sp = make_plan(g);
  StreamMaps maps;
  const void* ptrs[3] = {q, k, v};
  cudaError_t e = make_stream_maps(g, ptrs, &maps);
  if (e != cudaSuccess) return e;
  if (g.head_dim == 64)
    return out_f32 ? launch_s<64, true>(g, maps, sp, o, err, spin_limit, num_sms, stream)
                   : launch_s<64, false>(g, maps, sp, o, err, spin_limit, num_sms, stream);
  return out_f32 ? launch_s<32, true>(g, maps, sp, o, err, spin_limit, num_sms, stream)
                 : launch_s<32, false>(g, maps, sp, o, err, spin_limit, num_sms, stream);
}

}  // namespace s3w
