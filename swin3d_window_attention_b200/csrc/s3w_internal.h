// Host-side launch declarations shared between the C-ABI layer (api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>

#include "s3w_common.cuh"

namespace s3w {

// Window attention on the tcgen05 / TMEM path (attn_tcgen05.cu).
cudaError_t launch_window_attn_tc(const WinGeom& g, const void* q, const void* k, const void* v,
                                  void* o, bool out_f32, int* err, long long spin_limit,
                                  int num_sms, cudaStream_t stream);

// Arguments of the AdaLN half of the fused window attention + AdaLN kernel.
struct AdalnArgs {
  const float* residual;   // [B][L][C] fp32
  const float* scale;      // [B][C] fp32
  const float* shift;      // [B][C] fp32
  void* out;               // [B][L][C], fp32 or bf16; may be residual itself
  uint16_t* ws;            // workspace, per CTA 2 x 144 x C bf16 (window parity, slot, channel)
  float eps;
  int out_f32;
};

// Window attention fused with AdaLN + residual (attn_tcgen05.cu): o (bf16 attention output,
// grid layout) is optional (nullptr: not written).
cudaError_t launch_window_attn_adaln(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                     const AdalnArgs& fa, int* err, long long spin_limit, int num_sms,
                                     cudaStream_t stream);
// CTAs of the fused kernel (each takes whole windows); its workspace is grid x 2 x 144 x C bf16.
int window_attn_adaln_grid(long long windows, int num_sms);

// Window attention in the TF32_ACC_FP32 mode: fp32 Q/K/V, tcgen05 kind::tf32 (attn_tf32.cu).
cudaError_t launch_window_attn_tf32(const WinGeom& g, const void* q, const void* k, const void* v,
                                    void* o, bool out_f32, int* err, long long spin_limit,
                                    int num_sms, cudaStream_t stream);

// Window attention for windows of more than 144 slots (attn_stream.cu): BF16 Q/K/V, the
// window cut into blocks of whole (t, h) rows (<= 128 slots; win_w <= 128), K/V blocks
// streamed with online-softmax rescaling.  Units of work: windows x heads x blocks.
cudaError_t launch_window_attn_stream(const WinGeom& g, const void* q, const void* k, const void* v, void* o,
                                      bool out_f32, int* err, long long spin_limit, int num_sms,
                                      cudaStream_t stream);
long long window_attn_stream_units(const WinGeom& g);

// QKV projection (qkv_gemm.cu): qkv[l][n] = sum_c x[l][c] w[n][c] (+ bias[n]) for n < 3C, bf16
// in and out, fp32 accumulation, on the tensor cores.  x: [tokens][C], w: [3C][C], qkv:
// [tokens][3C]; C a multiple of 32.
cudaError_t launch_qkv_gemm(const void* x, const void* w, const float* bias, void* qkv, long long tokens, int C,
                            int* err, long long spin_limit, int num_sms, int test_stall, cudaStream_t stream);

// Window attention on the legacy warp-level mma.sync path (attn_mma.cu); kept as the
// measured baseline the tcgen05 kernel is compared with.
cudaError_t launch_window_attn_mma(const WinGeom& g, const void* q, const void* k, const void* v,
                                   void* o, bool out_f32, cudaStream_t stream);

// AdaLN + residual (adaln.cu).
cudaError_t launch_adaln(const void* x, bool x_bf16, const float* residual, const float* scale,
                         const float* shift, void* out, bool out_f32, int B, long long L, int C,
                         float eps, int num_sms, cudaStream_t stream);

}  // namespace s3w
