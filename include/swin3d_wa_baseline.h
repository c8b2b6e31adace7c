/*
 * swin3d_wa_baseline.h - the legacy-path baseline of the shifted-window attention library.
 *
 * Not a product entry point.  It computes exactly what swin3d_window_attn_fwd computes
 * (same arguments, checks and results; see swin3d_wa.h and the sections of "Flash-Aurora:
 * Toward Efficient Inference for Geospatial Foundation Models" cited there) on the legacy
 * warp-level tensor path: mma.sync, one CTA per (window, head), loads and math not
 * overlapped, no bounded waits.  It is exported so that the benchmark can time the path
 * the tcgen05 kernel replaces and the parity tests can check both against the oracle.
 */
#ifndef SWIN3D_WA_BASELINE_H_
#define SWIN3D_WA_BASELINE_H_

#include "swin3d_wa.h"

#ifdef __cplusplus
extern "C" {
#endif

int swin3d_window_attn_fwd_legacy_mma(const void* q, const void* k, const void* v, void* o,
                                      int B, int T, int H, int W,
                                      int win_t, int win_h, int win_w,
                                      int shift_t, int shift_h, int shift_w,
                                      int heads, int head_dim,
                                      long long qkv_token_stride, long long o_token_stride,
                                      float scale, int in_dtype, int out_dtype,
                                      s3w_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SWIN3D_WA_BASELINE_H_ */
