/*
 * swin3d_wa.h - C ABI of the B200 (sm_100a) Swin3D shifted-window attention path.
 *
 * Two compute calls, both asynchronous on the caller's CUDA stream:
 *
 *   swin3d_window_attn_fwd  cyclic shift + pad + 3D window partition, masked per-window
 *                           multi-head softmax attention, inverse merge + un-shift, all in
 *                           one kernel launch that reads Q/K/V straight from grid layout
 *                           and writes O straight back to grid layout.
 *   adaln_residual_fwd      LayerNorm + FiLM modulation + residual add in one pass, with
 *                           optional FP32 output.
 *
 * Defining passages ("Flash-Aurora: Toward Efficient Inference for Geospatial Foundation
 * Models"):
 *   - section "Kernel fusion for backbone memory traffic": cyclic shift, pad, 3D window
 *     partition and inverse merge fused instead of eager views/copies; LayerNorm, FiLM
 *     modulation and residual add without a full-width intermediate; FP32 activations
 *     between blocks (output_fp32).
 *   - section "CuTe DSL window attention": window (2,6,12) -> N = 144 tokens; logits
 *     S = scale * Q K^T, the Swin shift mask, row-wise softmax in FP32, O = softmax(S) V,
 *     no N x N map in global memory; BF16 activations with FP32 softmax (BF16_MIXED).
 *   - section "Window attention kernels": head_dim 64 on the production shapes.
 *
 * Semantics of swin3d_window_attn_fwd (the readings are stated where the pages leave a
 * step open):
 *   1. Each axis a of the token grid (T, H, W) is padded up to P_a = ceil(D_a / w_a) * w_a.
 *   2. The padded grid is rolled by -shift (pad first, then roll); window slot p' of
 *      axis a holds the original coordinate p = (p' + s_a) mod P_a; the token is real iff
 *      p < D_a on every axis.
 *   3. Region label per axis on the shifted grid: 0 if s_a = 0 or p' < P_a - w_a,
 *      1 if P_a - w_a <= p' < P_a - s_a, else 2.  Query i may attend key j iff j is real
 *      and the labels agree on every axis (the -infinity limit of Swin's -100 bias).
 *   4. Per (sample, window, head): S = scale * Q K^T (bf16 inputs, fp32 accumulate),
 *      masked softmax in fp32, the probabilities rounded to bf16, O = P V / rowsum(P)
 *      (fp32 accumulate).
 *   5. O of each real token is written to its original grid position, exactly once;
 *      padded slots are dropped.
 *
 * Memory layout: q, k, v and o are grid layout [B][T][H][W][token stride]; channel
 * c = head * head_dim + d.  The caller owns every buffer.  The library allocates no
 * device memory and keeps no state except a per-device error word and a cached SM count.
 *
 * Error convention: every argument check runs on the host before any launch; a failed
 * check returns a non-zero s3w_status and launches nothing.  A failed launch returns
 * S3W_ERR_CUDA.  A kernel whose bounded wait expired records S3W_ERR_DEVICE_TIMEOUT in
 * the device error word, which s3w_poll_device_error() reads and clears.
 */
#ifndef SWIN3D_WA_H_
#define SWIN3D_WA_H_

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* s3w_stream_t;

typedef enum {
  S3W_OK = 0,
  S3W_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, shift >= window, ...     */
  S3W_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim, window size, dtype combo   */
  S3W_ERR_MISALIGNED = 3,    /* pointer or stride not aligned as the call requires        */
  S3W_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed                      */
  S3W_ERR_DEVICE_TIMEOUT = 5 /* a bounded wait inside a kernel expired                    */
} s3w_status;

typedef enum { S3W_BF16 = 0, S3W_F32 = 1 } s3w_dtype;

/*
 * Shifted-window attention forward.
 *
 * Defines: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
 * section "CuTe DSL window attention" (per window and head: S = scale * Q K^T, the Swin
 * shift mask, softmax in FP32, O = softmax(S) V; window (2,6,12) -> N = 144; BF16_MIXED)
 * and section "Kernel fusion for backbone memory traffic" (cyclic shift, pad, 3D window
 * partition and the inverse merge folded into the kernel).  Semantics: steps 1-5 above.
 *
 * q, k, v   device pointers, in_dtype elements (S3W_BF16 only), grid layout with
 *           qkv_token_stride elements between consecutive tokens (>= heads*head_dim, a
 *           multiple of 8 so that every token row starts on a 16-byte boundary; q, k and v
 *           may be three slices of one fused [tokens][3C] buffer).  16-byte aligned.
 * o         device pointer, out_dtype elements (S3W_BF16 or S3W_F32), grid layout with
 *           o_token_stride elements between tokens (>= heads*head_dim, 16-byte rows).
 *           Must not overlap q, k or v (S3W_ERR_INVALID_ARG).  Channels beyond heads*head_dim
 *           are not written.
 * B,T,H,W   batch and unpadded grid sizes, each >= 1.
 * win_*     window extents, each >= 1, N = win_t*win_h*win_w.  1 <= N <= 144: one tile per
 *           (window, head).  144 < N <= 65536 (BF16 inputs, win_w <= 128): the streaming
 *           path of the same section (K/V blocks of whole (t, h) rows, <= 128 slots each,
 *           streamed past each query block with online-softmax rescaling).  Anything else
 *           returns S3W_ERR_UNSUPPORTED.
 * shift_*   0 <= shift < window on each axis.
 * heads     >= 1.  head_dim: 32 or 64.
 * scale     logit scale; a value <= 0 selects 1/sqrt(head_dim).
 * in_dtype, out_dtype  values of s3w_dtype, passed as int (the width of an enum is up to
 *           the compiler; int keeps the ABI fixed).
 * stream    CUDA stream; the call only enqueues work.
 *
 * Separate token strides for q/k/v and for o let q, k, v be slices of one fused QKV
 * buffer while o is a plain [tokens][C] tensor.
 *
 * Returns S3W_OK or an s3w_status; on error nothing is launched.
 */
int swin3d_window_attn_fwd(const void* q, const void* k, const void* v, void* o,
                           int B, int T, int H, int W,
                           int win_t, int win_h, int win_w,
                           int shift_t, int shift_h, int shift_w,
                           int heads, int head_dim,
                           long long qkv_token_stride, long long o_token_stride,
                           float scale, int in_dtype, int out_dtype,
                           s3w_stream_t stream);

/*
 * Fused AdaLN + residual forward.
 *
 * Defines: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
 * section "Kernel fusion for backbone memory traffic" (LayerNorm, FiLM modulation and the
 * residual add without a full-width intermediate) and section "Mixed-precision
 * inference" (FP32 activations between blocks, output_fp32).
 *
 * For every sample b and token l of x[B][L][C] (contiguous rows of C elements):
 *   mean = sum_c x / C,  var = sum_c (x - mean)^2 / C        (biased, two passes)
 *   out  = residual + (x - mean) / sqrt(var + eps) * (1 + scale[b]) + shift[b]
 * computed in fp32 and stored as out_dtype (S3W_F32 keeps the FP32 residual stream
 * between blocks; S3W_BF16 rounds to nearest even).
 *
 * x         device, x_dtype (S3W_BF16 or S3W_F32), [B][L][C], 16-byte aligned.
 * residual  device fp32 [B][L][C], 16-byte aligned.  out may alias residual exactly
 *           (in-place update of the residual stream); no other overlap is allowed.
 * scale, shift  device fp32 [B][C] per-sample FiLM vectors, 16-byte aligned.
 * out       device, out_dtype, [B][L][C], 16-byte aligned; must not overlap x, scale or
 *           shift (S3W_ERR_INVALID_ARG).
 * B >= 1, tokens_per_sample >= 0, C a multiple of 8 with 8 <= C <= 4096; eps >= 0.
 * With tokens_per_sample == 0 nothing is launched and the pointers are not used (they
 * may be NULL).  B * tokens_per_sample above (2^31 - 1) * 8 returns S3W_ERR_UNSUPPORTED.
 * x_dtype, out_dtype: values of s3w_dtype, passed as int.
 */
int adaln_residual_fwd(const void* x, int x_dtype, const float* residual,
                       const float* scale, const float* shift,
                       void* out, int out_dtype,
                       int B, long long tokens_per_sample, int C, float eps,
                       s3w_stream_t stream);

/*
 * Shifted-window attention fused with AdaLN + residual: one launch computes, for every token,
 *   x   = the window attention output of all heads (as swin3d_window_attn_fwd, rounded to
 *         bf16 exactly as that call stores it),
 *   out = residual + (x - mean) / sqrt(var + eps) * (1 + adaln_scale[b]) + adaln_shift[b]
 *         (as adaln_residual_fwd), without writing x to global memory in full.
 *
 * Defines: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
 * section "Kernel fusion for backbone memory traffic" (LayerNorm, FiLM modulation and the
 * residual add without a full-width intermediate; FP32 activations between blocks) with the
 * attention of section "CuTe DSL window attention" (BF16_MIXED).
 *
 * Each CTA takes whole windows, all heads of a window in a row, so every channel of a token
 * passes through one CTA.  The statistics of each token's row are merged head by head in
 * shared memory; the bf16 rows wait in `workspace` (per CTA, two windows deep) until the
 * window's last head is in, then the row is normalised and written to `out`.
 *
 * q, k, v, qkv_token_stride, the grid, window, shift, heads, head_dim (32 or 64) and
 *              attn_scale: as swin3d_window_attn_fwd; BF16 inputs only.
 * residual     device fp32 [B][T*H*W][C], C = heads * head_dim (C <= 4096), 32-byte aligned.
 * adaln_scale, adaln_shift  device fp32 [B][C], 32-byte aligned.
 * out          device, out_dtype (S3W_F32 or S3W_BF16), [B][T*H*W][C], 32-byte aligned; may
 *              alias residual exactly (in-place update of the residual stream); must not
 *              overlap q, k or v.
 * o            optional device bf16 [B][T][H][W][C] (token stride C), 32-byte aligned: when
 *              non-NULL the attention output is written there too; NULL skips it.  Must not
 *              overlap q, k or v.
 * workspace    device memory of at least swin3d_window_attn_adaln_workspace_bytes(...) bytes
 *              for the current device, 32-byte aligned, owned by the caller; its contents on
 *              entry do not matter.  Calls that overlap on the GPU must not share it.
 * eps          >= 0.
 * Returns S3W_OK or an s3w_status; on error nothing is launched.
 */
int swin3d_window_attn_adaln_fwd(const void* q, const void* k, const void* v, long long qkv_token_stride,
                                 const float* residual, const float* adaln_scale, const float* adaln_shift,
                                 void* out, int out_dtype, void* o, void* workspace, long long workspace_bytes,
                                 int B, int T, int H, int W,
                                 int win_t, int win_h, int win_w,
                                 int shift_t, int shift_h, int shift_w,
                                 int heads, int head_dim, float attn_scale, float eps,
                                 s3w_stream_t stream);

/*
 * Bytes of workspace swin3d_window_attn_adaln_fwd needs on the current device for this grid
 * (one CTA per SM up to the number of windows, 2 x 144 x C bf16 each).  A negative value is
 * minus an s3w_status (invalid sizes, or no CUDA device).
 */
long long swin3d_window_attn_adaln_workspace_bytes(int B, int T, int H, int W, int win_t, int win_h, int win_w,
                                                   int heads, int head_dim);

/* Size of the library's static workspace of swin3d_window_attn_adaln_fwd_static_ws: 48 MiB,
 * the two-window workspace of 148 CTAs at C = 512 (43.6 MB) with room to spare. */
#define S3W_ADALN_STATIC_WORKSPACE_BYTES (48ll << 20)

/*
 * swin3d_window_attn_adaln_fwd without a caller-supplied workspace, for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a deployment variant of
 * the fused call above, with the same arguments minus `workspace` and `workspace_bytes`, the
 * same semantics and the same results.
 *
 * The workspace is a file-scope device array of S3W_ADALN_STATIC_WORKSPACE_BYTES bytes in
 * the library (one per device, its address looked up once per device on first use).  The
 * array lives in a device-code module of its own, holding no kernels, so under CUDA's lazy
 * module loading (the default) it occupies device memory only on devices where this call
 * has run; with eager loading, on every device the process uses.  The call allocates nothing:
 * no cudaMalloc, no cudaFree, no allocating library routine.
 * Nothing in the array has to start at zero and the call clears nothing: every workspace
 * byte the kernel reads was written earlier in the same launch.
 *
 * Every call on a device shares the one array.  Calls that overlap on the GPU (on different
 * streams, or from different host threads without ordering between their streams) race on
 * it and their outputs are undefined; calls in one stream are ordered and safe.
 *
 * Returns S3W_ERR_UNSUPPORTED, launching nothing, when the grid needs more workspace than
 * the array holds (swin3d_window_attn_adaln_workspace_bytes(...) >
 * S3W_ADALN_STATIC_WORKSPACE_BYTES; e.g. C = 1024 on 148 SMs needs 87.3 MB), S3W_ERR_CUDA if
 * the array's address cannot be obtained, and otherwise what swin3d_window_attn_adaln_fwd
 * returns for the same arguments.
 */
int swin3d_window_attn_adaln_fwd_static_ws(const void* q, const void* k, const void* v, long long qkv_token_stride,
                                           const float* residual, const float* adaln_scale, const float* adaln_shift,
                                           void* out, int out_dtype, void* o,
                                           int B, int T, int H, int W,
                                           int win_t, int win_h, int win_w,
                                           int shift_t, int shift_h, int shift_w,
                                           int heads, int head_dim, float attn_scale, float eps,
                                           s3w_stream_t stream);

/*
 * QKV projection of grid-layout tokens, the prologue of the window attention:
 *   qkv[l][n] = sum_c x[l][c] * w_qkv[n][c] (+ b_qkv[n]),   n < 3C,
 * bf16 operands, fp32 accumulation on the tensor cores, bf16 output rounded to nearest even.
 * Features n = 0..C-1 are q, C..2C-1 are k, 2C..3C-1 are v, each in head-major order
 * (channel head * head_dim + d), the layout swin3d_window_attn_fwd reads with token stride 3C.
 *
 * Defines: "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation Models",
 * section "Mixed-precision inference" (bf16_mixed backbone: BF16 QKV projection feeding the
 * BF16 attention).
 *
 * x       device bf16 [tokens][C] (grid layout, contiguous), 16-byte aligned.
 * w_qkv   device bf16 [3C][C] (the Linear weight: output features x input channels), 16-byte
 *         aligned.
 * b_qkv   device fp32 [3C] or NULL (no bias), 16-byte aligned.
 * qkv     device bf16 [tokens][3C], 32-byte aligned, owned by the caller; must not overlap x,
 *         w_qkv or b_qkv.
 * tokens  1 .. 2^31 - 1.   C: a multiple of 32, <= 16384.
 * Returns S3W_OK or an s3w_status; on error nothing is launched.
 */
int swin3d_qkv_proj_fwd(const void* x, const void* w_qkv, const float* b_qkv, void* qkv, long long tokens, int C,
                        s3w_stream_t stream);

/*
 * The QKV projection followed by the shifted-window attention on its output: the attention
 * gathers its windows straight from the projection's grid-layout [tokens][3C] buffer (shift,
 * pad and partition folded into its loads), so no layout pass sits between the two launches.
 *
 * Defines: the two calls above ("Flash-Aurora: Toward Efficient Inference for Geospatial
 * Foundation Models", sections "Mixed-precision inference" and "Kernel fusion for backbone
 * memory traffic": no eager shift / pad / partition copies between projection and attention).
 *
 * x, w_qkv, b_qkv  as swin3d_qkv_proj_fwd, with C = heads * head_dim and tokens = B T H W.
 * qkv     device bf16 [B][T][H][W][3C] workspace (also an output: the projected q, k, v),
 *         32-byte aligned, owned by the caller.
 * o       device out_dtype (S3W_BF16 or S3W_F32) [B][T][H][W][C], token stride C; must not
 *         overlap qkv.
 * Grid, window, shift, heads, head_dim (32 or 64) and attn_scale: as swin3d_window_attn_fwd.
 * Every argument of both launches is checked before the first; on error nothing is launched.
 */
int swin3d_qkv_window_attn_fwd(const void* x, const void* w_qkv, const float* b_qkv, void* qkv, void* o,
                               int out_dtype, int B, int T, int H, int W,
                               int win_t, int win_h, int win_w,
                               int shift_t, int shift_h, int shift_w,
                               int heads, int head_dim, float attn_scale,
                               s3w_stream_t stream);

/* Static English text for a status code (never NULL). */
const char* s3w_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the calling device's error word.
 * Returns S3W_OK, S3W_ERR_DEVICE_TIMEOUT (a kernel gave up a bounded wait and returned
 * early; its output is incomplete) or S3W_ERR_CUDA (the synchronisation failed).
 */
int s3w_poll_device_error(s3w_stream_t stream);

/*
 * Time limit, in nanoseconds, of every bounded wait inside kernels launched after the
 * call (process-wide, safe to call from any thread); returns the previous limit.  Default 1e9 (one second).  With 0, a
 * wait not satisfied at its first poll expires: the kernel unwinds early (copies drained,
 * tensor memory released), records S3W_ERR_DEVICE_TIMEOUT in the device error word and
 * leaves the CUDA context usable.  Meant for tests of that failure path.
 */
long long s3w_set_wait_limit_ns(long long ns);

/*
 * Failure injection for tests (process-wide; returns the previous setting).  With a
 * nonzero value, every swin3d_window_attn_fwd launched after the call first waits on a
 * barrier that nothing signals, so that wait expires after the limit set above and the
 * kernel takes the timeout path (S3W_ERR_DEVICE_TIMEOUT in the error word, early exit,
 * context usable).  0 restores normal operation.  Nothing faults, traps or hangs: the
 * wait is bounded like every other one.
 */
int s3w_set_test_stall(int on);

/* Library version as major*10000 + minor*100 + patch. */
int s3w_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWIN3D_WA_H_ */
