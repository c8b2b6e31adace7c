// Shifted-window attention on the legacy warp-level tensor path (mma.sync m16n8k16,
// bf16 in, fp32 accumulate).  One CTA per (window, head), one warp per 16 query rows,
// S and P kept in registers.  This is the baseline the tcgen05 kernel is measured
// against; it shares the slot/label map with it (s3w_common.cuh).
//
// Method: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
// section "CuTe DSL window attention" (S = scale Q K^T, Swin mask, FP32 softmax,
// O = softmax(S) V, nothing N x N in global memory) and section "Kernel fusion for
// backbone memory traffic" (shift / pad / partition and the inverse merge are folded
// into the gather and the scatter here, so they never touch global memory).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s3w_internal.h"

namespace s3w {
namespace {

constexpr int kMaxN = 144;          // tokens per window supported by this kernel
constexpr int kMaxWarps = kMaxN / 16;

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int HD, bool OUT_F32>
__global__ void __launch_bounds__(kMaxWarps * 32)
window_attn_mma_kernel(WinGeom g, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                       const __nv_bfloat16* __restrict__ v, void* __restrict__ o) {
  constexpr int RS = HD + 8;               // padded smem row (elements): conflict-free ldmatrix
  constexpr int CH = HD / 8;               // 16-byte chunks per row
  constexpr int NT = kMaxN / 8;            // max key n-tiles
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + kMaxN * RS;
  __nv_bfloat16* sV = sK + kMaxN * RS;
  long long* sTok = reinterpret_cast<long long*>(sV + kMaxN * RS);
  int* sLab = reinterpret_cast<int*>(sTok + kMaxN);

  const long long tile = blockIdx.x;
  const long long win = tile / g.heads;
  const int head = static_cast<int>(tile - win * g.heads);
  const int NP = (g.N + 15) & ~15;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;

  for (int r = tid; r < NP; r += nthreads) {
    int lab = -1;
    long long tok = -1;
    if (r < g.N) {
      tok = slot_token(g, win, r, &lab);
      if (tok < 0) lab = -1;
    }
    sTok[r] = tok;
    sLab[r] = lab;
  }
  __syncthreads();

  // Gather: 16-byte cp.async straight from grid layout; padded slots are zero-filled.
  for (int i = tid; i < 3 * NP * CH; i += nthreads) {
    const int which = i / (NP * CH);
    const int rem = i - which * NP * CH;
    const int r = rem / CH, c = rem - (rem / CH) * CH;
    const long long tok = sTok[r];
    const __nv_bfloat16* base = which == 0 ? q : (which == 1 ? k : v);
    const __nv_bfloat16* src = base + (tok < 0 ? 0 : tok * g.qkv_stride + head * HD + c * 8);
    __nv_bfloat16* dstb = (which == 0 ? sQ : (which == 1 ? sK : sV)) + r * RS + c * 8;
    cp_async_16(smem_u32(dstb), src, tok >= 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();

  const int nwarps = NP / 16;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int row0 = warp * 16;
  float oacc[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
  float inv_l[2] = {0.f, 0.f};

  if (warp < nwarps) {
    uint32_t qa[HD / 16][4];
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk)
      ldsm_x4(smem_u32(sQ + (row0 + (lane & 15)) * RS + kk * 16 + (lane >> 4) * 8), qa[kk][0], qa[kk][1],
              qa[kk][2], qa[kk][3]);

    float s[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    // S = Q K^T, two key n-tiles per ldmatrix.x4
#pragma unroll
    for (int jp = 0; jp < NT / 2; ++jp) {
      if (jp * 16 < NP) {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          uint32_t b0, b1, b2, b3;
          const int key = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int d = kk * 16 + ((lane >> 3) & 1) * 8;
          ldsm_x4(smem_u32(sK + key * RS + d), b0, b1, b2, b3);
          mma_bf16(s[2 * jp], qa[kk], b0, b1);
          mma_bf16(s[2 * jp + 1], qa[kk], b2, b3);
        }
      }
    }
    // Mask (region label + padded keys), scale into log2 domain, row max.
    const int lab0 = sLab[row0 + g8], lab1 = sLab[row0 + g8 + 8];
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j * 8 < NP) {
        const int c0 = j * 8 + 2 * t4;
        const int lc0 = sLab[c0], lc1 = sLab[c0 + 1];
        s[j][0] = (lc0 >= 0 && lc0 == lab0) ? s[j][0] * g.scale_log2 : -INFINITY;
        s[j][1] = (lc1 >= 0 && lc1 == lab0) ? s[j][1] * g.scale_log2 : -INFINITY;
        s[j][2] = (lc0 >= 0 && lc0 == lab1) ? s[j][2] * g.scale_log2 : -INFINITY;
        s[j][3] = (lc1 >= 0 && lc1 == lab1) ? s[j][3] * g.scale_log2 : -INFINITY;
        m0 = fmaxf(m0, fmaxf(s[j][0], s[j][1]));
        m1 = fmaxf(m1, fmaxf(s[j][2], s[j][3]));
      }
    }
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
    if (m0 == -INFINITY) m0 = 0.f;  // row with no allowed key (padded query): all weights 0
    if (m1 == -INFINITY) m1 = 0.f;
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j * 8 < NP) {
        s[j][0] = exp2f(s[j][0] - m0);
        s[j][1] = exp2f(s[j][1] - m0);
        s[j][2] = exp2f(s[j][2] - m1);
        s[j][3] = exp2f(s[j][3] - m1);
        l0 += s[j][0] + s[j][1];
        l1 += s[j][2] + s[j][3];
      }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    inv_l[0] = l0 > 0.f ? 1.f / l0 : 0.f;
    inv_l[1] = l1 > 0.f ? 1.f / l1 : 0.f;

    // O = P V: the S accumulator layout of two adjacent key tiles is the A fragment.
#pragma unroll
    for (int kp = 0; kp < NT / 2; ++kp) {
      if (kp * 16 < NP) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(s[2 * kp][0], s[2 * kp][1]);
        pa[1] = pack_bf16x2(s[2 * kp][2], s[2 * kp][3]);
        pa[2] = pack_bf16x2(s[2 * kp + 1][0], s[2 * kp + 1][1]);
        pa[3] = pack_bf16x2(s[2 * kp + 1][2], s[2 * kp + 1][3]);
#pragma unroll
        for (int dn = 0; dn < HD / 8; dn += 2) {
          uint32_t b0, b1, b2, b3;
          const int key = kp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int d = (dn + (lane >> 4)) * 8;
          ldsm_x4_t(smem_u32(sV + key * RS + d), b0, b1, b2, b3);
          mma_bf16(oacc[dn], pa, b0, b1);
          mma_bf16(oacc[dn + 1], pa, b2, b3);
        }
      }
    }
  }
  __syncthreads();  // every warp is done with sK / sV: reuse them as the output stage

  // Stage this warp's 16 output rows (normalised, converted) then write 16-byte chunks.
  constexpr int OB = OUT_F32 ? 4 : 2;            // bytes per output element
  constexpr int ORB = HD * OB;                   // bytes per output row
  unsigned char* stage = reinterpret_cast<unsigned char*>(sK) + warp * 16 * ORB;
  if (warp < nwarps) {
#pragma unroll
    for (int dn = 0; dn < HD / 8; ++dn) {
      const int c = dn * 8 + 2 * t4;
      if constexpr (OUT_F32) {
        *reinterpret_cast<float2*>(stage + g8 * ORB + c * 4) = make_float2(oacc[dn][0] * inv_l[0], oacc[dn][1] * inv_l[0]);
        *reinterpret_cast<float2*>(stage + (g8 + 8) * ORB + c * 4) =
            make_float2(oacc[dn][2] * inv_l[1], oacc[dn][3] * inv_l[1]);
      } else {
        *reinterpret_cast<uint32_t*>(stage + g8 * ORB + c * 2) = pack_bf16x2(oacc[dn][0] * inv_l[0], oacc[dn][1] * inv_l[0]);
        *reinterpret_cast<uint32_t*>(stage + (g8 + 8) * ORB + c * 2) =
            pack_bf16x2(oacc[dn][2] * inv_l[1], oacc[dn][3] * inv_l[1]);
      }
    }
    __syncwarp();
    constexpr int CPR = ORB / 16;                // 16-byte chunks per row
    const int ob = OB;
    for (int i = lane; i < 16 * CPR; i += 32) {
      const int r = i / CPR, c = i - (i / CPR) * CPR;
      const int row = row0 + r;
      const long long tok = sTok[row];
      if (row < g.N && tok >= 0) {
        unsigned char* dst = reinterpret_cast<unsigned char*>(o) + (tok * g.o_stride + head * HD) * ob + c * 16;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(stage + r * ORB + c * 16);
      }
    }
  }
}

template <int HD, bool OUT_F32>
cudaError_t launch_t(const WinGeom& g, const void* q, const void* k, const void* v, void* o, cudaStream_t st) {
  constexpr int RS = HD + 8;
  const size_t smem = 3 * kMaxN * RS * sizeof(__nv_bfloat16) + kMaxN * (sizeof(long long) + sizeof(int));
  auto kern = window_attn_mma_kernel<HD, OUT_F32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long tiles = g.windows * g.heads;
  const int threads = ((g.N + 15) / 16) * 32;
  kern<<<static_cast<unsigned>(tiles), threads, smem, st>>>(
      g, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_attn_mma(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                   bool out_f32, cudaStream_t stream) {
  if (g.head_dim == 64)
    return out_f32 ? launch_t<64, true>(g, q, k, v, o, stream) : launch_t<64, false>(g, q, k, v, o, stream);
  return out_f32 ? launch_t<32, true>(g, q, k, v, o, stream) : launch_t<32, false>(g, q, k, v, o, stream);
}

}  // namespace s3w
