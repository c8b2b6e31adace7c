// QKV projection of grid-layout tokens on the sm_100a tensor cores, the prologue of the
// window attention: qkv[l][n] = sum_c x[l][c] w[n][c] + b[n] for every token l of the grid
// and n < 3C (the q, k and v features of every head, channel head * head_dim + d inside
// each third), bf16 operands, fp32 accumulation, bf16 out (round to nearest even).  The
// output stays in grid layout ([tokens][3C]), which is what the attention kernels gather
// their windows from (the shift, pad and partition are folded into their TMA loads), so no
// layout pass sits between the two.
//
// Method: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
// section "Mixed-precision inference" (bf16_mixed backbone: BF16 QKV projection feeding the
// BF16 CuTe attention) and section "Kernel fusion for backbone memory traffic" (no eager
// shift / pad / partition copies between the projection and the attention).
//
// Per CTA (persistent, one per SM), 10 warps:
//   warp 0   TMA: per output tile (128 tokens x 256 features) and K step of 64 channels, the
//            x box (64 x 128) and the w box (64 x 256) into a 3-stage ring, 128B swizzle.
//   warp 1   MMA: D (128 x 256, fp32, TMEM) += A B^T over 4 MMAs of K = 16 per stage; two
//            accumulators (512 TMEM columns) so tile i+1 accumulates while tile i drains.
//   warps 2-9 epilogue: warp w reads rows 32 (w % 4) .. of the accumulator (its TMEM lane
//            quarter) and the column half (w - 2) / 4, 64 columns per TMEM round trip, adds
//            the bias, rounds to bf16 and stores.  Eight warps drain a tile in the time the
//            MMAs of the next take (four, 32 columns at a time, were measured 7% slower).
// Every wait is bounded; a timeout unwinds the CTA (error word set, TMEM freed).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "attn_common.cuh"
#include "s3w_internal.h"
#include "sm100_ptx.cuh"

namespace s3w {
namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;      // tile: tokens x features x channels per stage
constexpr int kStagesG = 3;
constexpr int kABytes = kBM * kBK * 2;             // 16 KB
constexpr int kBBytes = kBN * kBK * 2;             // 32 KB
constexpr int kStageBytesG = kABytes + kBBytes;    // 48 KB
constexpr int kThreadsG = 320;
constexpr int kTmaWarpG = 0, kMmaWarpG = 1, kFirstEpiWarpG = 2;

struct SmemG {
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_BARS = kStagesG * kStageBytesG;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int kNumBars = 2 * kStagesG + 5;
  static constexpr int OFF_MISC = OFF_BARS + kNumBars * 8;   // tmem address, abort flag
  static constexpr int kBytes = OFF_MISC + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

struct GemmMaps {
  CUtensorMap x, w;
};

struct GemmGeom {
  long long tokens;   // rows of x and qkv
  int C;              // channels (K)
  int N;              // 3C features
  int ksteps;         // ceil(C / 64)
  int ntn;            // feature tiles: ceil(N / 256)
  long long tiles;    // ceil(tokens / 128) * ntn
  int test_stall;
};

template <int>
__global__ void __launch_bounds__(kThreadsG, 1)
qkv_gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmGeom gg,
                const float* __restrict__ bias, __nv_bfloat16* __restrict__ qkv, int* __restrict__ err,
                unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const uint32_t bar0 = sb + SmemG::OFF_BARS;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kStagesG + s); };
  auto acc_full = [&](int b) { return bar0 + 8u * (2 * kStagesG + b); };
  auto acc_empty = [&](int b) { return bar0 + 8u * (2 * kStagesG + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStagesG + 4);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm + SmemG::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SmemG::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long my_tiles =
      static_cast<long long>(blockIdx.x) < gg.tiles ? (gg.tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesG; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 256);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarpG) {
    tmem_alloc(sb + SmemG::OFF_MISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarpG) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.x);
      prefetch_tmap(&maps.w);
      long long it = 0;
      bool ok = true;
      for (long long i = 0; ok && i < my_tiles; ++i) {
        const long long t = blockIdx.x + i * gridDim.x;
        const long long m = t / gg.ntn;
        const int n = static_cast<int>(t - m * gg.ntn);
        for (int kk = 0; kk < gg.ksteps; ++kk, ++it) {
          const int s = static_cast<int>(it % kStagesG);
          if (*abort_flag ||
              !mbar_wait_bounded(empty(s), static_cast<uint32_t>(((it / kStagesG) & 1) ^ 1), limit_ns)) {
            ok = false;
            break;
          }
          const uint32_t st = sb + SmemG::OFF_STAGE + static_cast<uint32_t>(s * kStageBytesG);
          mbar_arrive_expect_tx(full(s), kStageBytesG);
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
              "[%4];" ::"r"(st),
              "l"(&maps.x), "r"(kk * kBK), "r"(static_cast<int>(m * kBM)), "r"(full(s))
              : "memory");
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
              "[%4];" ::"r"(st + kABytes),
              "l"(&maps.w), "r"(kk * kBK), "r"(n * kBN), "r"(full(s))
              : "memory");
        }
      }
      if (!ok) {
        record_error(err, kStatusTimeout);
        *abort_flag = 1;
      }
      // every load issued must land before the CTA exits (bounded)
      for (long long j = it > kStagesG ? it - kStagesG : 0; j < it; ++j)
        if (!mbar_wait_bounded(full(static_cast<int>(j % kStagesG)), static_cast<uint32_t>((j / kStagesG) & 1),
                               2000000000ull))
          record_error(err, kStatusTimeout);
    }
  } else if (warp == kMmaWarpG) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, false);
    const uint32_t leader = lane == 0 ? 1u : 0u;
    bool issued = false;
    bool ok = !gg.test_stall || __all_sync(0xffffffffu, mbar_wait_bounded(drain_bar, 0, limit_ns));
    long long it = 0;
    for (long long i = 0; ok && i < my_tiles; ++i) {
      const int ab = static_cast<int>(i & 1);
      if (__any_sync(0xffffffffu, *abort_flag != 0) ||
          !__all_sync(0xffffffffu,
                      mbar_wait_bounded(acc_empty(ab), static_cast<uint32_t>(((i >> 1) & 1) ^ 1), limit_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + static_cast<uint32_t>(ab * kBN);
      for (int kk = 0; kk < gg.ksteps; ++kk, ++it) {
        const int s = static_cast<int>(it % kStagesG);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full(s), static_cast<uint32_t>((it / kStagesG) & 1), limit_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = sb + SmemG::OFF_STAGE + static_cast<uint32_t>(s * kStageBytesG);
        const uint64_t a0 = smem_desc(st, 16, 1024, kSwizzle128B);
        const uint64_t b0 = smem_desc(st + kABytes, 16, 1024, kSwizzle128B);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          umma_bf16_ss_leader(d, a0 + 2 * k, b0 + 2 * k, idesc, (kk | k) ? 1u : 0u, leader);
        umma_commit_leader(empty(s), leader);
        issued = true;
      }
      if (!ok) break;
      umma_commit_leader(acc_full(ab), leader);
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
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;   // TMEM lane quarter: accumulator rows 32 q ..
    const int ch = (warp - kFirstEpiWarpG) >> 2;   // the tile's column half
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    bool aborted = false;
    for (long long i = 0; i < my_tiles; ++i) {
      const long long t = blockIdx.x + i * gridDim.x;
      const long long m = t / gg.ntn;
      const int n = static_cast<int>(t - m * gg.ntn);
      const int ab = static_cast<int>(i & 1);
      if (__any_sync(0xffffffffu, *abort_flag != 0) ||
          !__all_sync(0xffffffffu, mbar_wait_bounded(acc_full(ab), static_cast<uint32_t>((i >> 1) & 1), limit_ns))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const long long tok = m * kBM + q * 32 + lane;
      // the warp's column half, 64 columns per TMEM round trip, stored 32 at a time
#pragma unroll 1
      for (int c64 = ch * (kBN / 128); c64 < (ch + 1) * (kBN / 128); ++c64) {
        if (n * kBN + c64 * 64 >= gg.N) break;   // N is a multiple of 32
        float vv[64];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tmem_ld16(tmem + lane_base + static_cast<uint32_t>(ab * kBN + c64 * 64 + 16 * j), vv + 16 * j);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j) reg_fence16(vv + 16 * j);
        if (tok >= gg.tokens) continue;
#pragma unroll
        for (int c32 = 0; c32 < 2; ++c32) {
          const int f0 = n * kBN + c64 * 64 + c32 * 32;   // first feature of these 32
          if (f0 >= gg.N) break;
          float* v = vv + 32 * c32;
          if (bias != nullptr) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + f0 + e));
              v[e] += b4.x;
              v[e + 1] += b4.y;
              v[e + 2] += b4.z;
              v[e + 3] += b4.w;
            }
          }
          __nv_bfloat16* dst = qkv + tok * gg.N + f0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t u[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] = pack_bf16x2(v[16 * h + 2 * e], v[16 * h + 2 * e + 1]);
            st_global_v8(dst + 16 * h, u);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty(ab));
    }
    if (aborted) {
      if (lane == 0) record_error(err, kStatusTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarpG) tmem_dealloc(tmem, 512);
}

cudaError_t make_gemm_maps(const void* x, const void* w, long long tokens, int C, int N, GemmMaps* maps) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = attn::tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(tokens)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
    const cuuint32_t box[2] = {kBK, kBM};
    if (enc(&maps->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
    const cuuint32_t box[2] = {kBK, kBN};
    if (enc(&maps->w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_qkv_gemm(const void* x, const void* w, const float* bias, void* qkv, long long tokens, int C,
                            int* err, long long spin_limit, int num_sms, int test_stall, cudaStream_t stream) {
  GemmGeom gg;
  gg.tokens = tokens;
  gg.C = C;
  gg.N = 3 * C;
  gg.ksteps = (C + kBK - 1) / kBK;
  gg.ntn = (gg.N + kBN - 1) / kBN;
  gg.tiles = ((tokens + kBM - 1) / kBM) * gg.ntn;
  gg.test_stall = test_stall;
  GemmMaps maps;
  cudaError_t e = make_gemm_maps(x, w, tokens, C, gg.N, &maps);
  if (e != cudaSuccess) return e;
  auto kern = qkv_gemm_kernel<0>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemG::kAlloc);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(gg.tiles < num_sms ? gg.tiles : num_sms);
  kern<<<grid, kThreadsG, SmemG::kAlloc, stream>>>(maps, gg, bias, static_cast<__nv_bfloat16*>(qkv), err,
                                                   static_cast<unsigned long long>(spin_limit < 0 ? 0 : spin_limit));
  return cudaGetLastError();
}

}  // namespace s3w
