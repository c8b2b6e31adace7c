// Fused AdaLN + residual, one pass over global memory.
//
// "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models", section
// "Kernel fusion for backbone memory traffic": LayerNorm, FiLM modulation and the
// residual add without writing a full-width intermediate, with optional FP32 output so
// the next block reads FP32 residuals.  Per (sample b, token):
//   mean = sum(x)/C, var = sum((x-mean)^2)/C (biased, two passes over registers),
//   out  = residual + (x - mean) / sqrt(var + eps) * (1 + scale[b]) + shift[b].
//
// One warp per token row.  Each lane owns row chunks of 8 channels (16-byte loads of
// bf16 x, 2 x 16-byte loads of fp32 x / residual), keeps them in registers for both
// statistics passes and the output, and streams them with evict-first hints: every byte
// of x and residual is read once and every output byte written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s3w_internal.h"

namespace s3w {
namespace {

__device__ __forceinline__ float4 ld_stream_f4(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// NV = 8-channel chunks per lane (C <= 256 * NV).  With NV <= 8 the residual chunk is
// loaded together with x (more bytes in flight); wider rows load it in the output pass so
// the registers hold only x.
template <int NV, bool X_BF16, bool OUT_F32>
__global__ void __launch_bounds__(256)
adaln_residual_kernel(const void* __restrict__ x, const float* residual, const float* __restrict__ scale,
                      const float* __restrict__ shift, void* out, long long rows, long long L, int C, float eps) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const long long b = row / L;
  const int nchunk = C >> 3;
  constexpr bool kResEarly = NV <= 8;
  float xv[NV][8], rv[kResEarly ? NV : 1][8];
  const long long base = row * C;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int ch = lane + 32 * i;
    if (ch < nchunk) {
      const long long e = base + ch * 8;
      if constexpr (X_BF16) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + e));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h[j]);
          xv[i][2 * j] = f.x;
          xv[i][2 * j + 1] = f.y;
        }
      } else {
        const float4 a = ld_stream_f4(static_cast<const float*>(x) + e);
        const float4 c = ld_stream_f4(static_cast<const float*>(x) + e + 4);
        xv[i][0] = a.x; xv[i][1] = a.y; xv[i][2] = a.z; xv[i][3] = a.w;
        xv[i][4] = c.x; xv[i][5] = c.y; xv[i][6] = c.z; xv[i][7] = c.w;
      }
      if constexpr (kResEarly) {
        const float4 a = ld_stream_f4(residual + e);
        const float4 c = ld_stream_f4(residual + e + 4);
        rv[i][0] = a.x; rv[i][1] = a.y; rv[i][2] = a.z; rv[i][3] = a.w;
        rv[i][4] = c.x; rv[i][5] = c.y; rv[i][6] = c.z; rv[i][7] = c.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) xv[i][j] = 0.f;
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) s += xv[i][j];
  const float mean = warp_sum(s) / static_cast<float>(C);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    if (lane + 32 * i < nchunk) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = xv[i][j] - mean;
        ss = fmaf(d, d, ss);
      }
    }
  }
  const float var = warp_sum(ss) / static_cast<float>(C);
  const float rstd = 1.0f / sqrtf(var + eps);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int ch = lane + 32 * i;
    if (ch < nchunk) {
      const long long e = base + ch * 8;
      const float* scp = scale + b * C + ch * 8;
      const float* shp = shift + b * C + ch * 8;
      const float4 sc0 = __ldg(reinterpret_cast<const float4*>(scp));
      const float4 sc1 = __ldg(reinterpret_cast<const float4*>(scp + 4));
      const float4 sh0 = __ldg(reinterpret_cast<const float4*>(shp));
      const float4 sh1 = __ldg(reinterpret_cast<const float4*>(shp + 4));
      const float scv[8] = {sc0.x, sc0.y, sc0.z, sc0.w, sc1.x, sc1.y, sc1.z, sc1.w};
      const float shv[8] = {sh0.x, sh0.y, sh0.z, sh0.w, sh1.x, sh1.y, sh1.z, sh1.w};
      float r8[8];
      if constexpr (kResEarly) {
#pragma unroll
        for (int j = 0; j < 8; ++j) r8[j] = rv[i][j];
      } else {
        const float4 a = ld_stream_f4(residual + e);
        const float4 c = ld_stream_f4(residual + e + 4);
        r8[0] = a.x; r8[1] = a.y; r8[2] = a.z; r8[3] = a.w;
        r8[4] = c.x; r8[5] = c.y; r8[6] = c.z; r8[7] = c.w;
      }
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = r8[j] + (xv[i][j] - mean) * rstd * (1.0f + scv[j]) + shv[j];
      if constexpr (OUT_F32) {
        float* op = static_cast<float*>(out) + e;
        __stcs(reinterpret_cast<float4*>(op), make_float4(y[0], y[1], y[2], y[3]));
        __stcs(reinterpret_cast<float4*>(op + 4), make_float4(y[4], y[5], y[6], y[7]));
      } else {
        uint4 u;
        u.x = pack_bf16x2(y[0], y[1]);
        u.y = pack_bf16x2(y[2], y[3]);
        u.z = pack_bf16x2(y[4], y[5]);
        u.w = pack_bf16x2(y[6], y[7]);
        __stcs(reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + e), u);
      }
    }
  }
}

template <int NV>
cudaError_t launch_nv(const void* x, bool x_bf16, const float* res, const float* sc, const float* sh, void* out,
                      bool out_f32, long long rows, long long L, int C, float eps, cudaStream_t st) {
  const int rows_per_block = 8;
  const long long blocks = (rows + rows_per_block - 1) / rows_per_block;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (x_bf16) {
    if (out_f32)
      adaln_residual_kernel<NV, true, true><<<grid, 256, 0, st>>>(x, res, sc, sh, out, rows, L, C, eps);
    else
      adaln_residual_kernel<NV, true, false><<<grid, 256, 0, st>>>(x, res, sc, sh, out, rows, L, C, eps);
  } else {
    if (out_f32)
      adaln_residual_kernel<NV, false, true><<<grid, 256, 0, st>>>(x, res, sc, sh, out, rows, L, C, eps);
    else
      adaln_residual_kernel<NV, false, false><<<grid, 256, 0, st>>>(x, res, sc, sh, out, rows, L, C, eps);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_adaln(const void* x, bool x_bf16, const float* residual, const float* scale, const float* shift,
                         void* out, bool out_f32, int B, long long L, int C, float eps, int /*num_sms*/,
                         cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * L;
  if (rows == 0) return cudaSuccess;
  const int nchunk = C / 8;
  if (nchunk <= 32) return launch_nv<1>(x, x_bf16, residual, scale, shift, out, out_f32, rows, L, C, eps, stream);
  if (nchunk <= 64) return launch_nv<2>(x, x_bf16, residual, scale, shift, out, out_f32, rows, L, C, eps, stream);
  if (nchunk <= 128) return launch_nv<4>(x, x_bf16, residual, scale, shift, out, out_f32, rows, L, C, eps, stream);
  if (nchunk <= 256) return launch_nv<8>(x, x_bf16, residual, scale, shift, out, out_f32, rows, L, C, eps, stream);
  return launch_nv<16>(x, x_bf16, residual, scale, shift, out, out_f32, rows, L, C, eps, stream);
}

}  // namespace s3w
