// Pieces shared by the two tensor-core window-attention kernels (BF16 operands in
// attn_tcgen05.cu, TF32 operands in attn_tf32.cu): the per-tile slot tables and key masks,
// the tile -> (sample, window, head) decode, the TMA tensor maps and the two producer roles
// (the TMA loader and the table writer).
//
// Geometry ("Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
// section "Kernel fusion for backbone memory traffic"): each axis is padded to a multiple of
// the window and the padded grid is rolled by -shift; slot (rt, rh, rw) of the window whose
// first slot sits at shifted coordinate (bt, bh, bw) holds the original coordinate
// (b + r + s) mod P on each axis, real iff inside the unpadded grid.  The mask (section
// "CuTe DSL window attention", Swin's shifted-window mask) keeps key j for query i iff j is
// real and, on every axis where the window is the last one of a shifted axis, both lie on
// the same side of the wrap-around split.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "s3w_common.cuh"
#include "sm100_ptx.cuh"

namespace s3w {
namespace attn {

using namespace sm100;

constexpr int kN = 144;          // slots per window tile (queries and keys)
constexpr int kRowBytes = 128;   // one token row of one 128-byte channel chunk in shared memory
constexpr int kChunkTileBytes = kN * kRowBytes;   // 18432: one channel chunk of one tensor
constexpr int kMaskWords = 5;    // 144 key bits

// Per tile: grid token of every slot (-1 = padded), which slots are real, and along which
// shifted axes the window is the last one (where Swin's mask splits it in two regions).
struct Table {
  int tok[kN];
  uint32_t real[kMaskWords];
  uint32_t last;
  // The key mask a softmax thread applies, per (region combination of the query, key half):
  // bytes 0..8 = key groups 2k + half (k = 0..8), one bit per key; w = 1 if any key is masked.
  uint4 maskq[16];
};
constexpr int kTableBytes = (static_cast<int>(sizeof(Table)) + 15) & ~15;
// Per CTA, the same for every tile: the (t, h, w) offset of each slot inside the window
// and, per axis, the slots of the wrapped-around part (offset >= window - shift).  A query
// in the last window along a shifted axis may only see keys on its own side of that split.
struct SlotConst {
  uint32_t coord[kN];                 // rt | rh << 8 | rw << 16
  uint32_t hi[3][kMaskWords];
  uint32_t all[kMaskWords];           // slots < N
};
constexpr int kSlotConstBytes = (static_cast<int>(sizeof(SlotConst)) + 15) & ~15;

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Keys visible to a query in slot r: real slots, restricted on every axis where the window
// is the last one of a shifted axis to the query's side of the wrap-around split.
// hi_bits: bit a set iff slot r is in the wrapped-around part of axis a.
__device__ __forceinline__ void build_mask(const Table& tb, const SlotConst& sc, uint32_t last, uint32_t hi_bits,
                                           uint32_t (&m)[kMaskWords]) {
#pragma unroll
  for (int w = 0; w < kMaskWords; ++w) {
    uint32_t x = tb.real[w];
#pragma unroll
    for (int a = 0; a < 3; ++a)
      if ((last >> a) & 1u) x &= ((hi_bits >> a) & 1u) ? sc.hi[a][w] : (sc.all[w] & ~sc.hi[a][w]);
    m[w] = x;
  }
}

// Per-CTA slot constants, written by threads 0..143, 160..174 and 192..196.
__device__ __forceinline__ void init_slot_consts(const WinGeom& g, SlotConst* slotc, int tid) {
  auto split_at = [&](int a) { return a == 0 ? g.wt - g.st : (a == 1 ? g.wh - g.sh : g.ww - g.sw); };
  // offset of slot r along axis a.  Slots run T-slab by T-slab; inside a slab, h-major rows of
  // w, except that with a W shift each slab holds first the rows of the w offsets before the
  // wrap-around split (win_w - shift_w of them), then the rows of the rest.  The split is where
  // a window cut by the W seam wraps, so every slab loads in whole boxes (see the loader).
  auto slot_off = [&](int r, int a) {
    const int per_slab = g.ww * g.wh;
    const int rt = r / per_slab, i = r - rt * per_slab;
    if (a == 0) return rt;
    int rh, rw;
    if (g.sw > 0) {
      const int n1 = g.ww - g.sw;
      if (i < g.wh * n1) {
        rh = i / n1;
        rw = i - rh * n1;
      } else {
        const int j = i - g.wh * n1;
        rh = j / g.sw;
        rw = n1 + (j - rh * g.sw);
      }
    } else {
      rh = i / g.ww;
      rw = i - rh * g.ww;
    }
    return a == 1 ? rh : rw;
  };
  if (tid < kN) slotc->coord[tid] = tid < g.N ? (slot_off(tid, 0) | slot_off(tid, 1) << 8 | slot_off(tid, 2) << 16) : 0u;
  if (tid >= 160 && tid < 160 + 3 * kMaskWords) {
    const int a = (tid - 160) / kMaskWords, w = (tid - 160) % kMaskWords;
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b) {
      const int r = 32 * w + b;
      if (r < g.N && slot_off(r, a) >= split_at(a)) bits |= 1u << b;
    }
    slotc->hi[a][w] = bits;
  }
  if (tid >= 192 && tid < 192 + kMaskWords) {
    const int w = tid - 192;
    uint32_t bits = 0;
    for (int b = 0; b < 32; ++b)
      if (32 * w + b < g.N) bits |= 1u << b;
    slotc->all[w] = bits;
  }
}

// Window coordinates of a tile (32-bit: the tile count is checked on the host) and the
// shifted padded coordinate of its slot offset 0 plus the shift: slot (rt, rh, rw) holds
// the original coordinate (base + offset) mod P on each axis.
struct TileCoord {
  int head, bsmp, itw, ih, iw, bt, bh, bw;
};
__device__ __forceinline__ TileCoord tile_coord(const WinGeom& g, long long tile) {
  TileCoord tc;
  const int t32 = static_cast<int>(tile);
  const int win = fdiv(t32, g.div_heads);
  tc.head = t32 - win * g.heads;
  tc.bsmp = fdiv(win, g.div_per_sample);
  const int rem = win - tc.bsmp * (g.nwt * g.nwh * g.nww);
  const int q1 = fdiv(rem, g.div_nww);
  tc.iw = rem - q1 * g.nww;
  tc.itw = fdiv(q1, g.div_nwh);
  tc.ih = q1 - tc.itw * g.nwh;
  tc.bt = tc.itw * g.wt + g.st;
  tc.bh = tc.ih * g.wh + g.sh;
  tc.bw = tc.iw * g.ww + g.sw;
  return tc;
}

// Tensor maps of Q, K and V over the grid as a 5-D tensor (channel, W, H, T, sample),
// one per box shape.  A window is loaded one T-slab (win_h x win_w tokens) at a time.
// Without a W shift: the whole slab in one box, or, where the window wraps around the H
// seam, in two (win_h - shift_h rows, then shift_h rows).  With a W shift the slab's slots
// hold part A (the first n1 = win_w - shift_w offsets of every row) and then part B (the
// other shift_w), each h-major; A and B are one box each (two each at the H seam).  The
// W seam of a window always falls between A and B, so no window needs more boxes.
// Every box is one 128-byte channel chunk wide (64 bf16 or 32 fp32 channels), 128-byte
// swizzle, out-of-bounds elements (padding) read as zero.
enum : int {
  kBoxSlab = 0,     // win_w x win_h
  kBoxSeamH1 = 1,   // win_w x (win_h - shift_h)
  kBoxSeamH2 = 2,   // win_w x shift_h
  kBoxA = 3,        // n1 x win_h
  kBoxB = 4,        // shift_w x win_h
  kBoxA1 = 5,       // n1 x (win_h - shift_h)
  kBoxA2 = 6,       // n1 x shift_h
  kBoxB1 = 7,       // shift_w x (win_h - shift_h)
  kBoxB2 = 8,       // shift_w x shift_h
  kBoxShapes = 9
};
struct TmaMaps {
  CUtensorMap m[3][kBoxShapes];   // [tensor q/k/v][box shape]
};

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult qres;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// fp32 = true: 4-byte elements (32-channel boxes), else bf16 (64-channel boxes).  With
// v_atom32, V is written with the 128-byte swizzle of 32-byte chunks (4-row pattern), the
// layout the tensor core reads a 4-byte MN-major operand in.
inline cudaError_t make_maps(const WinGeom& g, const void* const ptrs[3], bool fp32, TmaMaps* maps,
                             bool v_atom32 = false) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t es = fp32 ? 4 : 2;
  const cuuint64_t C = static_cast<cuuint64_t>(g.heads) * g.head_dim;
  const cuuint64_t dims[5] = {C, static_cast<cuuint64_t>(g.W), static_cast<cuuint64_t>(g.H),
                              static_cast<cuuint64_t>(g.T), static_cast<cuuint64_t>(g.B)};
  const cuuint64_t row = static_cast<cuuint64_t>(g.qkv_stride) * es;
  const cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, row * g.W * g.H * g.T};
  // box (W, H) extents per shape; a shape of an unshifted axis is never used and gets the
  // whole window's extent instead
  const cuuint32_t ww = static_cast<cuuint32_t>(g.ww), wh = static_cast<cuuint32_t>(g.wh);
  const cuuint32_t sw = static_cast<cuuint32_t>(g.sw), sh = static_cast<cuuint32_t>(g.sh);
  const cuuint32_t n1 = ww - sw, n2 = sw > 0 ? sw : ww, h1 = wh - sh, h2 = sh > 0 ? sh : wh;
  const cuuint32_t boxwh[kBoxShapes][2] = {{ww, wh}, {ww, h1}, {ww, h2}, {n1, wh}, {n2, wh},
                                           {n1, h1}, {n1, h2}, {n2, h1}, {n2, h2}};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const cuuint32_t box_c = static_cast<cuuint32_t>(kRowBytes / es);
  // Only the shapes the loader can use for this geometry are encoded (host time per call);
  // the others are copies of the first one used, valid maps that no load names.
  bool used[kBoxShapes] = {};
  if (sw == 0) {
    used[kBoxSlab] = true;
    used[kBoxSeamH1] = used[kBoxSeamH2] = sh > 0;
  } else {
    used[kBoxA] = used[kBoxB] = true;
    used[kBoxA1] = used[kBoxA2] = used[kBoxB1] = used[kBoxB2] = sh > 0;
  }
  const int first = sw == 0 ? kBoxSlab : kBoxA;
  for (int t = 0; t < 3; ++t) {
    for (int b = 0; b < kBoxShapes; ++b) {
      if (!used[b]) continue;
      const cuuint32_t box[5] = {box_c, boxwh[b][0], boxwh[b][1], 1, 1};
      CUresult r = enc(&maps->m[t][b], fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                       const_cast<void*>(ptrs[t]), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       (t == 2 && v_atom32) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    for (int b = 0; b < kBoxShapes; ++b)
      if (!used[b]) maps->m[t][b] = maps->m[t][first];
  }
  return cudaSuccess;
}

// The CTA's it-th tile, or -1 when it has none left.  Strided order (WINDOW_MAJOR false):
// tile = blockIdx.x + it * gridDim.x.  Window-major order: the CTA takes whole windows,
// window blockIdx.x + (it / heads) * gridDim.x, all its heads in a row (tile = window *
// heads + head), so that every head of a token's row passes through one CTA.
template <bool WINDOW_MAJOR>
__device__ __forceinline__ long long cta_tile(const WinGeom& g, int it) {
  if constexpr (!WINDOW_MAJOR) {
    const long long t = blockIdx.x + static_cast<long long>(it) * gridDim.x;
    return t < g.windows * g.heads ? t : -1;
  } else {
    const int k = fdiv(it, g.div_heads);
    const long long w = blockIdx.x + static_cast<long long>(k) * gridDim.x;
    return w < g.windows ? w * g.heads + (it - k * g.heads) : -1;
  }
}

// Shared-memory addresses of a ring of stages and its barriers (8 bytes each, consecutive).
struct Ring {
  uint32_t stage0;       // stage 0's Q tile
  uint32_t load_bar0;    // load[s]: the TMA thread's expect_tx arrival + the bytes
  uint32_t empty_bar0;   // empty[s]: the stage may be refilled
  uint32_t table_bar0;   // table[s]: the stage's table is written
};

// TMA loader (one thread).  Per tile: wait until the stage is free, then load Q, K and V of
// the tile's (sample, window, head), CHUNKS channel chunks of 128 bytes (CHUNK_CH channels)
// per token row, in the boxes of the tensor maps above (per T-slab: one, or two parts A and
// B with a W shift, each cut in two at the H seam), straight from grid layout into the
// stage: tensor x, chunk c at stage + x * CHUNKS * kChunkTileBytes + c * kChunkTileBytes,
// rows in slot order.  Padded coordinates are out of bounds and read as zero.  On an abort, or after the
// last tile, waits (bounded) for the loads still in flight before returning.
template <int CHUNKS, int CHUNK_CH, int STAGES, int STAGE_BYTES, bool WINDOW_MAJOR = false>
__device__ __forceinline__ void tma_loader(const WinGeom& g, const TmaMaps& maps, const Ring& ring, int head_dim,
                                           long long num_tiles, volatile int* abort_flag, int* err,
                                           unsigned long long limit_ns) {
  constexpr int kTensorBytes = CHUNKS * kChunkTileBytes;
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < kBoxShapes; ++b) prefetch_tmap(&maps.m[a][b]);
  const uint32_t tile_bytes = static_cast<uint32_t>(3 * CHUNKS * g.N * kRowBytes);
  const uint32_t run_bytes = static_cast<uint32_t>(g.ww) * kRowBytes;
  int it = 0;
  for (long long tile = cta_tile<WINDOW_MAJOR>(g, 0); tile >= 0 && tile < num_tiles;
       tile = cta_tile<WINDOW_MAJOR>(g, ++it)) {
    const int s = it % STAGES;
    if (*abort_flag) break;
    if (!mbar_wait_bounded(ring.empty_bar0 + 8u * s, ((it / STAGES) & 1) ^ 1, limit_ns)) {
      record_error(err, kStatusTimeout);
      *abort_flag = 1;
      break;
    }
    const TileCoord tc = tile_coord(g, tile);
    const uint32_t stage = ring.stage0 + s * STAGE_BYTES;
    const uint32_t bar = ring.load_bar0 + 8u * s;
    mbar_arrive_expect_tx(bar, tile_bytes);
    // The window's first slot sits at (bt, bh, bw), inside the padded grid on every
    // axis; a window wraps around an axis's seam only if it is the last one along a
    // shifted axis.  n1h rows come before the H seam, the rest after it.
    const bool wrap_h = tc.bh + g.wh > g.Ph;
    const int n1h = g.Ph - tc.bh;
    const int n1 = g.ww - g.sw;
    int xb = tc.bw + n1;          // part B's first w (0 where the window wraps around the W seam)
    xb -= xb >= g.Pw ? g.Pw : 0;
#pragma unroll 1
    for (int rt = 0; rt < g.wt; ++rt) {
      int t = tc.bt + rt;
      t -= t >= g.Pt ? g.Pt : 0;
      const uint32_t slab = stage + rt * g.wh * run_bytes;
#pragma unroll 1
      for (int tsr = 0; tsr < 3; ++tsr) {
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
          const uint32_t d = slab + tsr * kTensorBytes + c * kChunkTileBytes;
          const int c0 = tc.head * head_dim + c * CHUNK_CH;
          const CUtensorMap* m = maps.m[tsr];
          if (g.sw == 0) {
            if (!wrap_h) {
              tma_load_5d(d, &m[kBoxSlab], c0, tc.bw, tc.bh, t, tc.bsmp, bar);
            } else {
              tma_load_5d(d, &m[kBoxSeamH1], c0, tc.bw, tc.bh, t, tc.bsmp, bar);
              tma_load_5d(d + n1h * run_bytes, &m[kBoxSeamH2], c0, tc.bw, 0, t, tc.bsmp, bar);
            }
          } else {
            const uint32_t db = d + static_cast<uint32_t>(g.wh * n1) * kRowBytes;   // part B
            if (!wrap_h) {
              tma_load_5d(d, &m[kBoxA], c0, tc.bw, tc.bh, t, tc.bsmp, bar);
              tma_load_5d(db, &m[kBoxB], c0, xb, tc.bh, t, tc.bsmp, bar);
            } else {
              tma_load_5d(d, &m[kBoxA1], c0, tc.bw, tc.bh, t, tc.bsmp, bar);
              tma_load_5d(d + static_cast<uint32_t>(n1h * n1) * kRowBytes, &m[kBoxA2], c0, tc.bw, 0, t, tc.bsmp,
                          bar);
              tma_load_5d(db, &m[kBoxB1], c0, xb, tc.bh, t, tc.bsmp, bar);
              tma_load_5d(db + static_cast<uint32_t>(n1h * g.sw) * kRowBytes, &m[kBoxB2], c0, xb, 0, t, tc.bsmp,
                          bar);
            }
          }
        }
      }
    }
  }
  // Before the CTA may exit, every load issued must have landed.  On the normal path the
  // MMA warp has consumed them all; after an abort, wait (bounded, independently of the
  // test limit) for the last stages issued.
  for (int j = it > STAGES ? it - STAGES : 0; j < it; ++j)
    if (!mbar_wait_bounded(ring.load_bar0 + 8u * (j % STAGES), (j / STAGES) & 1, 2000000000ull))
      record_error(err, kStatusTimeout);
}

// Table writer (one warp, named barrier 1).  Per tile, once the stage is free: the slot ->
// grid-token map, the bitmask of real slots, the "last window along a shifted axis" flags
// and, from these, the key masks per (region combination, key half).
template <int STAGES, bool WINDOW_MAJOR = false>
__device__ __forceinline__ void table_writer(const WinGeom& g, Table* tables, const SlotConst* slotc, const Ring& ring,
                                             long long num_tiles, volatile int* abort_flag, volatile int* prod_stop,
                                             int* err, unsigned long long limit_ns, int lane) {
  int it = 0;
  for (long long tile = cta_tile<WINDOW_MAJOR>(g, 0); tile >= 0 && tile < num_tiles;
       tile = cta_tile<WINDOW_MAJOR>(g, ++it)) {
    const int s = it % STAGES;
    if (lane == 0) {
      const bool ok = mbar_wait_bounded(ring.empty_bar0 + 8u * s, ((it / STAGES) & 1) ^ 1, limit_ns);
      if (!ok) {
        record_error(err, kStatusTimeout);
        *abort_flag = 1;
      }
      *prod_stop = (!ok || *abort_flag) ? 1 : 0;
    }
    named_bar_sync(1, 32);
    if (*prod_stop) break;
    const TileCoord tc = tile_coord(g, tile);
    auto resolve = [&](int r) -> int {   // grid token of slot r, -1 if padded
      if (r >= g.N) return -1;
      const uint32_t cd = slotc->coord[r];
      int t = tc.bt + static_cast<int>(cd & 0xffu);
      int h = tc.bh + static_cast<int>((cd >> 8) & 0xffu);
      int w = tc.bw + static_cast<int>(cd >> 16);
      t -= t >= g.Pt ? g.Pt : 0;
      h -= h >= g.Ph ? g.Ph : 0;
      w -= w >= g.Pw ? g.Pw : 0;
      if (t >= g.T || h >= g.H || w >= g.W) return -1;
      return ((tc.bsmp * g.T + t) * g.H + h) * g.W + w;
    };
    Table& tb = tables[s];
#pragma unroll 1
    for (int r = lane; r < kN; r += 32) tb.tok[r] = resolve(r);
    if (lane == 0)
      tb.last = ((tc.itw == g.nwt - 1 && g.st > 0) ? 1u : 0u) | ((tc.ih == g.nwh - 1 && g.sh > 0) ? 2u : 0u) |
                ((tc.iw == g.nww - 1 && g.sw > 0) ? 4u : 0u);
#pragma unroll 1
    for (int wd = 0; wd < kMaskWords; ++wd) {
      const int r = 32 * wd + lane;
      const unsigned m = __ballot_sync(0xffffffffu, r < kN && resolve(r) >= 0);
      if (lane == 0) tb.real[wd] = m;
    }
    __syncwarp();
    if (lane < 16) {
      // combination c of the query's wrapped-around sides (bit a: axis a), key half h
      const uint32_t c = static_cast<uint32_t>(lane) >> 1, h = static_cast<uint32_t>(lane) & 1u;
      uint32_t mw[kMaskWords];
      build_mask(tb, *slotc, tb.last, c, mw);
      uint32_t kb[9];
#pragma unroll
      for (int k = 0; k < 9; ++k) kb[k] = (mw[k >> 1] >> (16 * (k & 1) + 8 * h)) & 0xffu;
      const uint32_t all = kb[0] & kb[1] & kb[2] & kb[3] & kb[4] & kb[5] & kb[6] & kb[7] & kb[8];
      tb.maskq[lane] = make_uint4(kb[0] | kb[1] << 8 | kb[2] << 16 | kb[3] << 24,
                                  kb[4] | kb[5] << 8 | kb[6] << 16 | kb[7] << 24, kb[8], all == 0xffu ? 0u : 1u);
    }
    mbar_arrive(ring.table_bar0 + 8u * s);   // table written (release)
  }
}

// Epilogue store of the softmax threads: a thread holds HD / 2 outputs of one query row, the
// column groups 32 m + 16 half .. +15 (m < HD / 32), in v[16 m + j], scaled here by inv and
// written to token `tok` (-1: a padded slot, nothing written) of grid tensor o.  Every lane of
// the warp calls it; the lanes of a pair (2i, 2i+1) hold rows of the same key half.
//  * bf16, HD = 64, 32-byte rows: the thread's two 32-byte pieces sit 64 bytes apart in one
//    128-byte line.  The lanes of a pair swap one piece each, so the first store instruction
//    writes both pieces of the even lane's row and the second those of the odd lane's row: 16
//    lines per warp instruction instead of 32 (the store path's cost is per line).
//  * otherwise, 32-byte rows: one 32-byte store per 16 bf16 or 8 fp32 values.
//  * rows not 32-byte aligned: 16-byte stores.
template <int HD, bool OUT_F32>
__device__ __forceinline__ void store_o_row(void* o, long long o_stride, bool rows_32b, int tok, int head, int half,
                                            int lane, const float* v, float inv) {
  constexpr int kGroups = HD / 32 > 0 ? HD / 32 : 1;
  constexpr int kPer = HD >= 32 ? 16 : HD / 2;   // values per column group
  if constexpr (!OUT_F32 && HD == 64) {
    if (rows_32b) {
      uint32_t u0[8], u1[8], x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        u0[e] = pack_bf16x2(v[2 * e] * inv, v[2 * e + 1] * inv);
        u1[e] = pack_bf16x2(v[16 + 2 * e] * inv, v[16 + 2 * e + 1] * inv);
      }
      const bool odd = lane & 1;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __shfl_xor_sync(0xffffffffu, odd ? u0[e] : u1[e], 1);
      const int ptok = __shfl_xor_sync(0xffffffffu, tok, 1);
      const int t1 = odd ? ptok : tok, t2 = odd ? tok : ptok;
      __nv_bfloat16* base = static_cast<__nv_bfloat16*>(o) + head * HD + (odd ? 32 : 0) + 16 * half;
      if (t1 >= 0) sm100::st_global_v8(base + static_cast<long long>(t1) * o_stride, odd ? x : u0);
      if (t2 >= 0) sm100::st_global_v8(base + static_cast<long long>(t2) * o_stride, odd ? u1 : x);
      return;
    }
  }
  if (tok < 0) return;
#pragma unroll
  for (int m = 0; m < kGroups; ++m) {
    const int col = 32 * m + 16 * half;
    const float* w = v + 16 * m;
    if constexpr (OUT_F32) {
      float* dst = static_cast<float*>(o) + static_cast<long long>(tok) * o_stride + head * HD + col;
#pragma unroll
      for (int q = 0; q < kPer; q += 8) {
        if (rows_32b && kPer % 8 == 0) {
          uint32_t u[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) u[e] = __float_as_uint(w[q + e] * inv);
          sm100::st_global_v8(dst + q, u);
        } else {
#pragma unroll
          for (int r = 0; r < 8 && q + r < kPer; r += 4)
            *reinterpret_cast<float4*>(dst + q + r) =
                make_float4(w[q + r] * inv, w[q + r + 1] * inv, w[q + r + 2] * inv, w[q + r + 3] * inv);
        }
      }
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o) + static_cast<long long>(tok) * o_stride + head * HD + col;
      if (rows_32b && kPer == 16) {
        uint32_t u[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) u[e] = pack_bf16x2(w[2 * e] * inv, w[2 * e + 1] * inv);
        sm100::st_global_v8(dst, u);
      } else {
#pragma unroll
        for (int q = 0; q < kPer; q += 8) {
          uint4 u;
          u.x = pack_bf16x2(w[q] * inv, w[q + 1] * inv);
          u.y = pack_bf16x2(w[q + 2] * inv, w[q + 3] * inv);
          u.z = pack_bf16x2(w[q + 4] * inv, w[q + 5] * inv);
          u.w = pack_bf16x2(w[q + 6] * inv, w[q + 7] * inv);
          *reinterpret_cast<uint4*>(dst + q) = u;
        }
      }
    }
  }
}

}  // namespace attn
}  // namespace s3w
