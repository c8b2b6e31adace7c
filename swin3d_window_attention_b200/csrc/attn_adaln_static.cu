// The fused attention + AdaLN call for callers that cannot allocate device memory: the
// workspace of swin3d_window_attn_adaln_fwd is a file-scope device array of a fixed size,
// shared by every call on a device.  The call allocates nothing; it checks the size the
// grid needs against the array and then makes the ordinary fused call with the array as
// its workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "swin3d_wa.h"

namespace {

constexpr long long kStaticWorkspaceBytes = S3W_ADALN_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

// The fused kernel writes every workspace byte it reads earlier in the same launch, so the
// array needs no clearing, at load time or between calls.
static __device__ __align__(256) unsigned char g_adaln_static_workspace[kStaticWorkspaceBytes];

void* g_workspace[kMaxDevices];
std::mutex g_mu;

// Device address of the array on the current device, looked up once per device.
int static_workspace(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return S3W_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_workspace[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_adaln_static_workspace) != cudaSuccess || p == nullptr) return S3W_ERR_CUDA;
    g_workspace[dev] = p;
  }
  *ptr = g_workspace[dev];
  return S3W_OK;
}

}  // namespace

extern "C" {

int swin3d_window_attn_adaln_fwd_static_ws(const void* q, const void* k, const void* v, long long qkv_token_stride,
                                           const float* residual, const float* adaln_scale, const float* adaln_shift,
                                           void* out, int out_dtype, void* o, int B, int T, int H, int W, int win_t,
                                           int win_h, int win_w, int shift_t, int shift_h, int shift_w, int heads,
                                           int head_dim, float attn_scale, float eps, s3w_stream_t stream) {
  const long long need = swin3d_window_attn_adaln_workspace_bytes(B, T, H, W, win_t, win_h, win_w, heads, head_dim);
  if (need < 0) return static_cast<int>(-need);
  if (need > kStaticWorkspaceBytes) return S3W_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const int rc = static_workspace(&ws);
  if (rc != S3W_OK) return rc;
  return swin3d_window_attn_adaln_fwd(q, k, v, qkv_token_stride, residual, adaln_scale, adaln_shift, out, out_dtype,
                                      o, ws, kStaticWorkspaceBytes, B, T, H, W, win_t, win_h, win_w, shift_t, shift_h,
                                      shift_w, heads, head_dim, attn_scale, eps, stream);
}

}  // extern "C"
