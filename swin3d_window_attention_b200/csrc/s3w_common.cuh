// Shared device-side pieces of the window-attention kernels: window geometry, the
// slot -> grid-token map of the cyclic shift / pad / partition, the Swin region label,
// and the device error word.
//
// Geometry follows "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation
// Models", section "Kernel fusion for backbone memory traffic" (cyclic shift, pad, 3D
// window partition, inverse merge), read as: pad each axis to a multiple of the window,
// roll the padded grid by -shift, cut windows.  Slot p' of an axis holds the original
// coordinate (p' + s) mod P; the token is real iff that coordinate is inside the grid.
// The mask of section "CuTe DSL window attention" (Swin's shifted-window mask) keeps
// key j for query i iff j is real and both carry the same region label, where the label
// of an axis is 0 / 1 / 2 for slots in [0, P-w), [P-w, P-s), [P-s, P) when s > 0.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace s3w {

enum : int { kStatusTimeout = 5 };

// Division by a runtime-invariant divisor d >= 1 for 0 <= n < 2^31 by one 64-bit multiply
// and a shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with l = ceil(log2 d) and m = ceil(2^(31+l) / d),
// n / d = (n * m) >> (31 + l).  The host computes (m, l).
struct FastDiv {
  uint32_t m;
  int shift;   // 31 + l
};
inline FastDiv make_fastdiv(uint32_t d) {
  int l = 0;
  while ((1ull << l) < d) ++l;
  const unsigned long long num = 1ull << (31 + l);
  FastDiv f;
  f.m = static_cast<uint32_t>((num + d - 1) / d);
  f.shift = 31 + l;
  return f;
}
__host__ __device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  return static_cast<int>((static_cast<unsigned long long>(static_cast<uint32_t>(n)) * f.m) >> f.shift);
}

// Everything a kernel needs to map (window id, slot) to a grid token.  Passed by value.
struct WinGeom {
  int B, T, H, W;          // unpadded grid
  int wt, wh, ww;          // window
  int st, sh, sw;          // shift
  int Pt, Ph, Pw;          // padded grid
  int nwt, nwh, nww;       // windows per axis
  int N;                   // tokens per window
  int heads, head_dim;
  long long windows;       // B * nwt * nwh * nww
  long long qkv_stride;    // elements between tokens in q/k/v
  long long o_stride;      // elements between tokens in o
  float scale_log2;        // scale * log2(e)
  int o_rows_32b;          // 1 if every output row start is 32-byte aligned
  FastDiv div_heads, div_per_sample, div_nww, div_nwh;   // tile -> (sample, window, head)
  int test_stall;          // failure injection: first wait on a barrier nothing signals
};

// Per-axis region label on the shifted, padded grid.
__host__ __device__ __forceinline__ int axis_label(int pp, int P, int w, int s) {
  return (s == 0 || pp < P - w) ? 0 : (pp < P - s ? 1 : 2);
}

// Resolve slot r (0 <= r < N, row-major over (t, h, w) inside the window) of window
// `win` (flat over B and the window grid).  Returns the flat grid token index
// ((b*T + t)*H + h)*W + w, or -1 for a padded slot; *label gets the combined region label.
__host__ __device__ __forceinline__ long long slot_token(const WinGeom& g, long long win, int r, int* label) {
  const int per_sample = g.nwt * g.nwh * g.nww;
  const long long b = win / per_sample;
  int rem = static_cast<int>(win - b * per_sample);
  const int iw = rem % g.nww;
  rem /= g.nww;
  const int ih = rem % g.nwh;
  const int it = rem / g.nwh;
  const int rw = r % g.ww;
  const int rh = (r / g.ww) % g.wh;
  const int rt = r / (g.ww * g.wh);
  const int pt = it * g.wt + rt, ph = ih * g.wh + rh, pw = iw * g.ww + rw;  // shifted slots
  int t = pt + g.st, h = ph + g.sh, w = pw + g.sw;
  t -= (t >= g.Pt) ? g.Pt : 0;
  h -= (h >= g.Ph) ? g.Ph : 0;
  w -= (w >= g.Pw) ? g.Pw : 0;
  *label = axis_label(pt, g.Pt, g.wt, g.st) * 9 + axis_label(ph, g.Ph, g.wh, g.sh) * 3 +
           axis_label(pw, g.Pw, g.ww, g.sw);
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return ((b * g.T + t) * g.H + h) * g.W + w;
}

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace s3w
