// C ABI of the shifted-window attention library: host-side argument checks, the
// per-device error word, and kernel dispatch.  Every check runs before any launch; a
// failed check returns a status and enqueues nothing.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <climits>
#include <cstdint>
#include <mutex>

#include "swin3d_wa.h"
#include "swin3d_wa_baseline.h"
#include "s3w_internal.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr long long kMaxStreamN = 1 << 16;   // window slots on the streaming path

// One error word per device; kernels get its device address.
__device__ int g_s3w_error_word;

struct DeviceState {
  int* err = nullptr;
  int num_sms = 0;
  bool ready = false;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return S3W_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_s3w_error_word) != cudaSuccess) return S3W_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return S3W_ERR_CUDA;
    s.err = static_cast<int*>(p);
    s.num_sms = sms;
    s.ready = true;
  }
  *out = &s;
  return S3W_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Time limit of every bounded wait inside the kernels (nanoseconds); 1 s by default.  Both
// controls are process-wide and may be set from one host thread while another launches.
std::atomic<long long> g_wait_limit_ns{1000000000ll};
std::atomic<int> g_test_stall{0};

}  // namespace

extern "C" {

const char* s3w_status_string(int status) {
  switch (status) {
    case S3W_OK: return "ok";
    case S3W_ERR_INVALID_ARG: return "invalid argument";
    case S3W_ERR_UNSUPPORTED: return "unsupported configuration";
    case S3W_ERR_MISALIGNED: return "pointer or stride not aligned as the call requires";
    case S3W_ERR_CUDA: return "CUDA runtime error";
    case S3W_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel expired";
    default: return "unknown status";
  }
}

int s3w_version(void) { return 100; }

int s3w_poll_device_error(s3w_stream_t stream) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return S3W_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ds->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return S3W_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpy(ds->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return S3W_ERR_CUDA;
    return S3W_ERR_DEVICE_TIMEOUT;
  }
  return S3W_OK;
}

}  // extern "C"

namespace {

// True when the byte range [p, p + bytes) meets any of the q, k, v token ranges (tokens rows of
// row_bytes at a stride of stride_bytes).  The callers bound every size below 2^62.
bool overlaps_qkv(const void* q, const void* k, const void* v, long long stride_bytes, long long row_bytes,
                  long long tokens, const void* p, long long bytes) {
  const char* p0 = static_cast<const char*>(p);
  const char* p1 = p0 + bytes;
  for (const void* t : {q, k, v}) {
    const char* t0 = static_cast<const char*>(t);
    const char* t1 = t0 + (tokens - 1) * stride_bytes + row_bytes;
    if (p0 < t1 && t0 < p1) return true;
  }
  return false;
}

// Host-side checks shared by both attention entry points; fills the kernel geometry.
int make_geometry(const void* q, const void* k, const void* v, void* o, int B, int T, int H, int W, int win_t,
                  int win_h, int win_w, int shift_t, int shift_h, int shift_w, int heads, int head_dim,
                  long long qkv_token_stride, long long o_token_stride, float scale, int in_dtype, int out_dtype,
                  s3w::WinGeom* out) {
  if (!q || !k || !v || !o) return S3W_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || head_dim < 1) return S3W_ERR_INVALID_ARG;
  if (win_t < 1 || win_h < 1 || win_w < 1) return S3W_ERR_INVALID_ARG;
  if (shift_t < 0 || shift_h < 0 || shift_w < 0 || shift_t >= win_t || shift_h >= win_h || shift_w >= win_w)
    return S3W_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return S3W_ERR_INVALID_ARG;
  if ((in_dtype != S3W_BF16 && in_dtype != S3W_F32) || (out_dtype != S3W_BF16 && out_dtype != S3W_F32))
    return S3W_ERR_INVALID_ARG;
  const long long C = static_cast<long long>(heads) * head_dim;
  if (qkv_token_stride < C || o_token_stride < C) return S3W_ERR_INVALID_ARG;
  if (win_t > 65536 || win_h > 65536 || win_w > 65536) return S3W_ERR_UNSUPPORTED;   // keeps N in range
  const long long N = static_cast<long long>(win_t) * win_h * win_w;
  // N <= 144: one tile per (window, head); above, the streaming kernel, whose blocks hold
  // whole rows of win_w tokens (<= 128), and only for BF16 inputs
  if (N > 144 && (win_w > 128 || in_dtype != S3W_BF16 || N > kMaxStreamN)) return S3W_ERR_UNSUPPORTED;
  if (head_dim != 32 && head_dim != 64) return S3W_ERR_UNSUPPORTED;
  const int ib = in_dtype == S3W_F32 ? 4 : 2;
  const int ob = out_dtype == S3W_F32 ? 4 : 2;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return S3W_ERR_MISALIGNED;
  if ((qkv_token_stride * ib) % 16 != 0 || (o_token_stride * ob) % 16 != 0) return S3W_ERR_MISALIGNED;
  // grid token indices are 32-bit inside the kernels; padded sizes must stay in int range
  if (static_cast<long long>(B) * T * H * W > INT32_MAX) return S3W_ERR_UNSUPPORTED;
  const long long Pt = (T + win_t - 1) / win_t * static_cast<long long>(win_t);
  const long long Ph = (H + win_h - 1) / win_h * static_cast<long long>(win_h);
  const long long Pw = (W + win_w - 1) / win_w * static_cast<long long>(win_w);
  if (Pt > INT32_MAX / 2 || Ph > INT32_MAX / 2 || Pw > INT32_MAX / 2) return S3W_ERR_UNSUPPORTED;
  const long long per_sample = (Pt / win_t) * (Ph / win_h) * (Pw / win_w);
  if (per_sample > INT32_MAX) return S3W_ERR_UNSUPPORTED;
  if (per_sample * B * heads > INT32_MAX) return S3W_ERR_UNSUPPORTED;  // tile index is 32-bit
  // streaming path: units = tiles x blocks (at most win_t x win_h blocks per window)
  if (N > 144 && per_sample * B * heads * win_t * win_h > INT32_MAX) return S3W_ERR_UNSUPPORTED;
  // o must not overlap q, k or v (which may overlap one another: slices of one buffer).  The
  // sizes are bounded above (tokens < 2^31, strides checked against C), so no product overflows
  // once the strides are below 2^31.
  if (qkv_token_stride > INT32_MAX || o_token_stride > INT32_MAX) return S3W_ERR_UNSUPPORTED;
  {
    const long long tokens = static_cast<long long>(B) * T * H * W;
    if (overlaps_qkv(q, k, v, qkv_token_stride * ib, C * ib, tokens, o, ((tokens - 1) * o_token_stride + C) * ob))
      return S3W_ERR_INVALID_ARG;
  }

  s3w::WinGeom& g = *out;
  g = s3w::WinGeom{};
  g.B = B; g.T = T; g.H = H; g.W = W;
  g.wt = win_t; g.wh = win_h; g.ww = win_w;
  g.st = shift_t; g.sh = shift_h; g.sw = shift_w;
  g.Pt = static_cast<int>(Pt); g.Ph = static_cast<int>(Ph); g.Pw = static_cast<int>(Pw);
  g.nwt = g.Pt / win_t; g.nwh = g.Ph / win_h; g.nww = g.Pw / win_w;
  g.N = static_cast<int>(N);
  g.heads = heads;
  g.head_dim = head_dim;
  g.windows = per_sample * B;
  g.qkv_stride = qkv_token_stride;
  g.o_stride = o_token_stride;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(head_dim));
  g.scale_log2 = sc * 1.4426950408889634f;  // log2(e): the softmax is evaluated with exp2
  g.o_rows_32b = ((reinterpret_cast<uintptr_t>(o) & 31u) == 0 && (o_token_stride * ob) % 32 == 0) ? 1 : 0;
  g.div_heads = s3w::make_fastdiv(static_cast<uint32_t>(heads));
  g.div_per_sample = s3w::make_fastdiv(static_cast<uint32_t>(per_sample));
  g.div_nww = s3w::make_fastdiv(static_cast<uint32_t>(g.nww));
  g.div_nwh = s3w::make_fastdiv(static_cast<uint32_t>(g.nwh));
  return S3W_OK;
}

}  // namespace

extern "C" {

long long s3w_set_wait_limit_ns(long long ns) {
  return g_wait_limit_ns.exchange(ns < 0 ? 0 : ns, std::memory_order_relaxed);
}

int s3w_set_test_stall(int on) { return g_test_stall.exchange(on ? 1 : 0, std::memory_order_relaxed); }

int swin3d_window_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int T, int H, int W,
                           int win_t, int win_h, int win_w, int shift_t, int shift_h, int shift_w, int heads,
                           int head_dim, long long qkv_token_stride, long long o_token_stride, float scale,
                           int in_dtype, int out_dtype, s3w_stream_t stream) {
  s3w::WinGeom g;
  int rc = make_geometry(q, k, v, o, B, T, H, W, win_t, win_h, win_w, shift_t, shift_h, shift_w, heads, head_dim,
                         qkv_token_stride, o_token_stride, scale, in_dtype, out_dtype, &g);
  if (rc != S3W_OK) return rc;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  g.test_stall = g_test_stall.load(std::memory_order_relaxed);
  const long long limit = g_wait_limit_ns.load(std::memory_order_relaxed);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e =
      g.N > 144 ? s3w::launch_window_attn_stream(g, q, k, v, o, out_dtype == S3W_F32, ds->err, limit, ds->num_sms, st)
      : in_dtype == S3W_F32
          ? s3w::launch_window_attn_tf32(g, q, k, v, o, out_dtype == S3W_F32, ds->err, limit, ds->num_sms, st)
          : s3w::launch_window_attn_tc(g, q, k, v, o, out_dtype == S3W_F32, ds->err, limit, ds->num_sms, st);
  return e == cudaSuccess ? S3W_OK : S3W_ERR_CUDA;
}

int swin3d_window_attn_fwd_legacy_mma(const void* q, const void* k, const void* v, void* o, int B, int T, int H,
                                      int W, int win_t, int win_h, int win_w, int shift_t, int shift_h, int shift_w,
                                      int heads, int head_dim, long long qkv_token_stride, long long o_token_stride,
                                      float scale, int in_dtype, int out_dtype, s3w_stream_t stream) {
  s3w::WinGeom g;
  int rc = make_geometry(q, k, v, o, B, T, H, W, win_t, win_h, win_w, shift_t, shift_h, shift_w, heads, head_dim,
                         qkv_token_stride, o_token_stride, scale, in_dtype, out_dtype, &g);
  if (rc != S3W_OK) return rc;
  if (in_dtype != S3W_BF16) return S3W_ERR_UNSUPPORTED;   // the baseline path is BF16 only
  if (g.N > 144) return S3W_ERR_UNSUPPORTED;               // and single-tile windows only
  if (g.windows * heads > (1ll << 31) - 1) return S3W_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  cudaError_t e = s3w::launch_window_attn_mma(g, q, k, v, o, out_dtype == S3W_F32,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? S3W_OK : S3W_ERR_CUDA;
}

long long swin3d_window_attn_adaln_workspace_bytes(int B, int T, int H, int W, int win_t, int win_h, int win_w,
                                                  int heads, int head_dim) {
  if (B < 1 || T < 1 || H < 1 || W < 1 || win_t < 1 || win_h < 1 || win_w < 1 || heads < 1 || head_dim < 1)
    return -S3W_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  const int rc = device_state(&ds);
  if (rc != S3W_OK) return -rc;
  const long long windows = static_cast<long long>(B) * ((T + win_t - 1) / win_t) * ((H + win_h - 1) / win_h) *
                            ((W + win_w - 1) / win_w);
  const long long grid = s3w::window_attn_adaln_grid(windows, ds->num_sms);
  return grid * 2 * 144 * static_cast<long long>(heads) * head_dim * 2;
}

int swin3d_window_attn_adaln_fwd(const void* q, const void* k, const void* v, long long qkv_token_stride,
                                 const float* residual, const float* adaln_scale, const float* adaln_shift,
                                 void* out, int out_dtype, void* o, void* workspace, long long workspace_bytes,
                                 int B, int T, int H, int W, int win_t, int win_h, int win_w, int shift_t,
                                 int shift_h, int shift_w, int heads, int head_dim, float attn_scale, float eps,
                                 s3w_stream_t stream) {
  if (!residual || !adaln_scale || !adaln_shift || !out || !workspace) return S3W_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || std::isinf(eps)) return S3W_ERR_INVALID_ARG;
  if (out_dtype != S3W_BF16 && out_dtype != S3W_F32) return S3W_ERR_INVALID_ARG;
  const long long C = static_cast<long long>(heads) * head_dim;
  // attention checks (o, when given, is a bf16 grid tensor with token stride C)
  s3w::WinGeom g;
  int rc = make_geometry(q, k, v, o ? o : out, B, T, H, W, win_t, win_h, win_w, shift_t, shift_h, shift_w, heads,
                         head_dim, qkv_token_stride, C, attn_scale, S3W_BF16, S3W_BF16, &g);
  if (rc != S3W_OK) return rc;
  if (g.N > 144) return S3W_ERR_UNSUPPORTED;   // the fused kernel takes single-tile windows
  if (C % 8 != 0 || C > 4096) return S3W_ERR_UNSUPPORTED;
  // the AdaLN part moves 32-byte vectors of every one of these
  auto aligned32 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; };
  if (!aligned32(residual) || !aligned32(adaln_scale) || !aligned32(adaln_shift) || !aligned32(out) ||
      !aligned32(workspace) || (o && !aligned32(o)))
    return S3W_ERR_MISALIGNED;
  // out may alias residual exactly; any other overlap with residual is rejected
  const long long n = static_cast<long long>(B) * T * H * W * C;
  const char* r0 = reinterpret_cast<const char*>(residual);
  const char* o0 = reinterpret_cast<const char*>(out);
  const long long ob = out_dtype == S3W_F32 ? 4 : 2;
  if (o0 != r0 && o0 < r0 + n * 4 && r0 < o0 + n * ob) return S3W_ERR_INVALID_ARG;
  // out is written while other windows still read q, k and v
  if (overlaps_qkv(q, k, v, qkv_token_stride * 2, C * 2, n / C, out, n * ob)) return S3W_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  const long long grid = s3w::window_attn_adaln_grid(g.windows, ds->num_sms);
  if (workspace_bytes < grid * 2 * 144 * C * 2) return S3W_ERR_INVALID_ARG;
  g.test_stall = g_test_stall.load(std::memory_order_relaxed);
  s3w::AdalnArgs fa{residual, adaln_scale, adaln_shift, out, static_cast<uint16_t*>(workspace), eps,
                    out_dtype == S3W_F32 ? 1 : 0};
  cudaError_t e = s3w::launch_window_attn_adaln(g, q, k, v, o, fa, ds->err,
                                                g_wait_limit_ns.load(std::memory_order_relaxed), ds->num_sms,
                                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? S3W_OK : S3W_ERR_CUDA;
}

int swin3d_qkv_proj_fwd(const void* x, const void* w_qkv, const float* b_qkv, void* qkv, long long tokens, int C,
                        s3w_stream_t stream) {
  if (!x || !w_qkv || !qkv) return S3W_ERR_INVALID_ARG;
  if (tokens < 1 || C < 1) return S3W_ERR_INVALID_ARG;
  if (C % 32 != 0 || C > 16384) return S3W_ERR_UNSUPPORTED;
  if (tokens > INT32_MAX) return S3W_ERR_UNSUPPORTED;   // TMA row coordinates are 32-bit
  if (!aligned16(x) || !aligned16(w_qkv) || (b_qkv && !aligned16(b_qkv)) ||
      (reinterpret_cast<uintptr_t>(qkv) & 31u) != 0)
    return S3W_ERR_MISALIGNED;
  // qkv must not overlap x, w or the bias
  const char* q0 = static_cast<const char*>(qkv);
  const long long qbytes = tokens * 3 * C * 2;
  auto overlaps = [&](const void* p, long long bytes) {
    const char* a = static_cast<const char*>(p);
    return a < q0 + qbytes && q0 < a + bytes;
  };
  if (overlaps(x, tokens * C * 2) || overlaps(w_qkv, 3ll * C * C * 2) || (b_qkv && overlaps(b_qkv, 3ll * C * 4)))
    return S3W_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  cudaError_t e = s3w::launch_qkv_gemm(x, w_qkv, b_qkv, qkv, tokens, C, ds->err,
                                       g_wait_limit_ns.load(std::memory_order_relaxed), ds->num_sms,
                                       g_test_stall.load(std::memory_order_relaxed),
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? S3W_OK : S3W_ERR_CUDA;
}

int swin3d_qkv_window_attn_fwd(const void* x, const void* w_qkv, const float* b_qkv, void* qkv, void* o,
                               int out_dtype, int B, int T, int H, int W, int win_t, int win_h, int win_w,
                               int shift_t, int shift_h, int shift_w, int heads, int head_dim, float attn_scale,
                               s3w_stream_t stream) {
  if (!x || !w_qkv || !qkv || !o) return S3W_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || head_dim < 1) return S3W_ERR_INVALID_ARG;
  const long long C = static_cast<long long>(heads) * head_dim;
  if (C > 16384) return S3W_ERR_UNSUPPORTED;
  // every check of the attention call first (geometry, dtypes, sizes: B T H W <= 2^31 - 1),
  // so that nothing is launched unless both launches are valid; the projection's follow
  s3w::WinGeom g;
  const char* qkvc = static_cast<const char*>(qkv);
  int rc = make_geometry(qkvc, qkvc + C * 2, qkvc + 2 * C * 2, o, B, T, H, W, win_t, win_h, win_w, shift_t, shift_h,
                         shift_w, heads, head_dim, 3 * C, C, attn_scale, S3W_BF16, out_dtype, &g);
  if (rc != S3W_OK) return rc;
  const long long tokens = static_cast<long long>(B) * T * H * W;
  // o must not overlap the projection's output, which the attention reads
  const char* o0 = static_cast<const char*>(o);
  const long long ob = out_dtype == S3W_F32 ? 4 : 2;
  if (o0 < qkvc + tokens * 3 * C * 2 && qkvc < o0 + tokens * C * ob) return S3W_ERR_INVALID_ARG;
  rc = swin3d_qkv_proj_fwd(x, w_qkv, b_qkv, qkv, tokens, static_cast<int>(C), stream);
  if (rc != S3W_OK) return rc;
  return swin3d_window_attn_fwd(qkvc, qkvc + C * 2, qkvc + 2 * C * 2, o, B, T, H, W, win_t, win_h, win_w, shift_t,
                                shift_h, shift_w, heads, head_dim, 3 * C, C, attn_scale, S3W_BF16, out_dtype, stream);
}

int adaln_residual_fwd(const void* x, int x_dtype, const float* residual, const float* scale, const float* shift,
                       void* out, int out_dtype, int B, long long tokens_per_sample, int C, float eps,
                       s3w_stream_t stream) {
  if (B < 1 || tokens_per_sample < 0 || C < 1 || !(eps >= 0.f) || std::isinf(eps)) return S3W_ERR_INVALID_ARG;
  if ((x_dtype != S3W_BF16 && x_dtype != S3W_F32) || (out_dtype != S3W_BF16 && out_dtype != S3W_F32))
    return S3W_ERR_INVALID_ARG;
  if (C % 8 != 0 || C > 4096) return S3W_ERR_UNSUPPORTED;
  if (tokens_per_sample == 0) return S3W_OK;  // nothing to read or write; pointers unused
  if (!x || !residual || !scale || !shift || !out) return S3W_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(residual) || !aligned16(scale) || !aligned16(shift) || !aligned16(out))
    return S3W_ERR_MISALIGNED;
  // One block of 8 rows each: the row count is bounded by the grid size limit (2^31 - 1
  // blocks); checked before any product that could overflow.
  constexpr long long kMaxRows = static_cast<long long>(INT32_MAX) * 8;
  if (tokens_per_sample > kMaxRows / B) return S3W_ERR_UNSUPPORTED;
  // out may alias residual exactly; any other overlap with residual is rejected
  const long long n = static_cast<long long>(B) * tokens_per_sample * C;
  const char* r0 = reinterpret_cast<const char*>(residual);
  const char* o0 = reinterpret_cast<const char*>(out);
  const long long ob = out_dtype == S3W_F32 ? 4 : 2;
  if (o0 != r0 && o0 < r0 + n * 4 && r0 < o0 + n * ob) return S3W_ERR_INVALID_ARG;
  // and out overlaps none of x, scale, shift
  auto meets_out = [&](const void* p, long long bytes) {
    const char* a = static_cast<const char*>(p);
    return a < o0 + n * ob && o0 < a + bytes;
  };
  if (meets_out(x, n * (x_dtype == S3W_F32 ? 4 : 2)) || meets_out(scale, B * 4ll * C) ||
      meets_out(shift, B * 4ll * C))
    return S3W_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != S3W_OK) return rc;
  cudaError_t e = s3w::launch_adaln(x, x_dtype == S3W_BF16, residual, scale, shift, out, out_dtype == S3W_F32, B,
                                    tokens_per_sample, C, eps, ds->num_sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? S3W_OK : S3W_ERR_CUDA;
}

}  // extern "C"
