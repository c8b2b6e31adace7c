// Plain, slow, fp64 CPU oracle for the Swin3D shifted-window attention path and the
// fused AdaLN + residual step of a Flash-Aurora-style backbone.
//
// TEST INFRASTRUCTURE ONLY.  This file is the yardstick the CUDA kernels are checked
// against; it is built and called only by the test suite, the smoke check and the
// CPU-baseline leg of the benchmark.  It shares no code, header, table or helper with
// the CUDA path, and the product path never links or calls it.
//
// Sources (page titles and sections):
//   [FA-fusion]  "Flash-Aurora: Toward Efficient Inference for Geospatial Foundation
//                Models", section "Kernel fusion for backbone memory traffic": cyclic
//                shift, pad, 3D window partition and the inverse merge; LayerNorm, FiLM
//                modulation and residual add fused, optional FP32 output.
//   [FA-attn]    same page, section "CuTe DSL window attention": logits S = scale*Q K^T,
//                optional Swin mask, row-wise softmax in FP32, O = softmax(S) V; window
//                (2,6,12) gives N = 144 tokens; the shift mask is the additive -100 bias
//                of PyTorch's Swin mask.
//   [FA-kernels] same page, section "Window attention kernels": (B, H, N, D_h) layout,
//                FP32 softmax.
//
// Readings where the pages leave a step open (each also listed in the design notes):
//   * pad first, then roll the padded grid by -shift; region labels live on the padded,
//     shifted grid (Swin's three slices per axis: [0,P-w), [P-w,P-s), [P-s,P));
//   * masked keys are excluded (the -infinity limit of the -100 bias); an additive -100
//     mode is kept to show the two agree to far below any tolerance;
//   * padded keys are excluded; padded queries are never written to the output;
//   * a shift is applied literally even on an axis no longer than its window;
//   * scale defaults to 1/sqrt(head_dim);
//   * AdaLN: out = residual + LN(x) * (1 + scale_b) + shift_b with LN = (x - mean) /
//     sqrt(var + eps), biased variance, no affine of its own.
//
// Every value is widened exactly to double before use; all arithmetic is double; no
// blocking, fusion or reordering beyond the definitions below.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// Element kinds of the input buffers.
enum InKind { IN_BF16 = 0, IN_F32 = 1, IN_F64 = 2 };

double widen(const void* base, int kind, int64_t idx) {
  if (kind == IN_BF16) {
    uint16_t h = static_cast<const uint16_t*>(base)[idx];
    uint32_t bits = static_cast<uint32_t>(h) << 16;
    float f;
    std::memcpy(&f, &bits, 4);
    return static_cast<double>(f);
  }
  if (kind == IN_F32) return static_cast<double>(static_cast<const float*>(base)[idx]);
  return static_cast<const double*>(base)[idx];
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Swin region label of one axis, from the coordinate on the padded, shifted grid
// [FA-fusion]: with no shift the whole axis is one region; otherwise the axis splits
// into [0, P-w), [P-w, P-s) and [P-s, P).
int axis_label(int64_t pprime, int64_t P, int64_t w, int64_t s) {
  if (s == 0) return 0;
  if (pprime < P - w) return 0;
  if (pprime < P - s) return 1;
  return 2;
}

struct Geometry {
  int64_t D[3], w[3], s[3], P[3], nwin[3];
  int64_t N, windows_per_sample;
};

Geometry make_geometry(int T, int H, int W, int wt, int wh, int ww, int st, int sh, int sw) {
  Geometry g;
  const int64_t D[3] = {T, H, W}, w[3] = {wt, wh, ww}, s[3] = {st, sh, sw};
  for (int a = 0; a < 3; ++a) {
    g.D[a] = D[a];
    g.w[a] = w[a];
    g.s[a] = s[a];
    g.P[a] = ceil_div(D[a], w[a]) * w[a];  // pad each axis up to a multiple of the window
    g.nwin[a] = g.P[a] / w[a];
  }
  g.N = g.w[0] * g.w[1] * g.w[2];
  g.windows_per_sample = g.nwin[0] * g.nwin[1] * g.nwin[2];
  return g;
}

}  // namespace

extern "C" {

int orc_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Shifted-window attention, one (sample, window) per listed id, all heads.
// [FA-fusion] shift/pad/partition and merge; [FA-attn] masked softmax attention.
//
// q, k, v : grid layout [B][T][H][W][token_stride], channel c = head*head_dim + d.
// window_ids : n_list ids, id = b * windows_per_sample + window (row-major over the
//              window counts along T, H, W); null means every window of every sample.
// out     : [n_list][N][heads*head_dim] doubles, in intra-window order (t, h, w
//           row-major); rows of padded tokens are left as NaN.
// out_tok : [n_list][N] flat grid index (((b*T + t)*H + h)*W + w) each row belongs to,
//           -1 for padded tokens.  The merge / un-shift is "row r goes to out_tok[r]".
// probs   : optional [n_list][heads][N][N] softmax weights (0 for masked pairs; rows of
//           padded queries are NaN).
// mask_mode : 0 excludes masked keys; 1 adds -100 to region-mismatch logits (padded keys
//           are excluded in both modes).
// Returns 0, or -1 on a bad argument.
int orc_window_attn(const void* q, const void* k, const void* v, int in_kind, int B, int T, int H,
                    int W, int wt, int wh, int ww, int st, int sh, int sw, int heads, int head_dim,
                    int64_t token_stride, double scale, int mask_mode, int64_t n_list,
                    const int64_t* window_ids, double* out, int64_t* out_tok, double* probs) {
  if (B < 1 || T < 1 || H < 1 || W < 1 || wt < 1 || wh < 1 || ww < 1 || heads < 1 || head_dim < 1)
    return -1;
  if (st < 0 || sh < 0 || sw < 0 || st >= wt || sh >= wh || sw >= ww) return -1;
  if (token_stride < static_cast<int64_t>(heads) * head_dim) return -1;
  const Geometry g = make_geometry(T, H, W, wt, wh, ww, st, sh, sw);
  const int64_t total_windows = g.windows_per_sample * B;
  if (window_ids == nullptr) n_list = total_windows;
  if (scale <= 0.0) scale = 1.0 / std::sqrt(static_cast<double>(head_dim));
  const int64_t N = g.N;
  const int64_t C = static_cast<int64_t>(heads) * head_dim;

  // Step 1 (per window): source coordinate, realness and region label of each token.
  // Done once per listed window, shared by all heads.
  std::vector<int64_t> tok(n_list * N);
  std::vector<int> label(n_list * N);
  for (int64_t li = 0; li < n_list; ++li) {
    const int64_t id = window_ids ? window_ids[li] : li;
    if (id < 0 || id >= total_windows) return -1;
    const int64_t b = id / g.windows_per_sample;
    int64_t rem = id % g.windows_per_sample;
    const int64_t wi[3] = {rem / (g.nwin[1] * g.nwin[2]), (rem / g.nwin[2]) % g.nwin[1],
                           rem % g.nwin[2]};
    for (int64_t r = 0; r < N; ++r) {
      const int64_t rr[3] = {r / (g.w[1] * g.w[2]), (r / g.w[2]) % g.w[1], r % g.w[2]};
      int64_t p[3];
      bool real = true;
      int lab = 0;
      for (int a = 0; a < 3; ++a) {
        const int64_t pprime = wi[a] * g.w[a] + rr[a];        // shifted, padded coordinate
        p[a] = (pprime + g.s[a]) % g.P[a];                      // where it came from
        real = real && (p[a] < g.D[a]);
        lab = lab * 3 + axis_label(pprime, g.P[a], g.w[a], g.s[a]);
      }
      tok[li * N + r] = real ? ((b * T + p[0]) * H + p[1]) * W + p[2] : -1;
      label[li * N + r] = lab;
    }
  }

  const double nan = std::nan("");
  for (int64_t i = 0; i < n_list * N * C; ++i) out[i] = nan;
  for (int64_t i = 0; i < n_list * N; ++i) out_tok[i] = tok[i];

  // Steps 2-5 per (window, head): logits, mask, softmax, weighted sum of V.
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t job = 0; job < n_list * heads; ++job) {
    const int64_t li = job / heads;
    const int64_t h = job % heads;
    const int64_t* t = &tok[li * N];
    const int* lab = &label[li * N];
    std::vector<double> logit(N), pw(N);
    for (int64_t i = 0; i < N; ++i) {
      if (t[i] < 0) {
        if (probs)
          for (int64_t j = 0; j < N; ++j) probs[((li * heads + h) * N + i) * N + j] = nan;
        continue;  // padded query: dropped on merge
      }
      const int64_t qi = t[i] * token_stride + h * head_dim;
      double m = -INFINITY;
      for (int64_t j = 0; j < N; ++j) {
        const bool key_real = t[j] >= 0;
        const bool same_region = lab[j] == lab[i];
        if (!key_real || (mask_mode == 0 && !same_region)) {
          logit[j] = -INFINITY;
          continue;
        }
        const int64_t kj = t[j] * token_stride + h * head_dim;
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d) dot += widen(q, in_kind, qi + d) * widen(k, in_kind, kj + d);
        logit[j] = scale * dot + ((mask_mode == 1 && !same_region) ? -100.0 : 0.0);
        if (logit[j] > m) m = logit[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        pw[j] = (logit[j] == -INFINITY) ? 0.0 : std::exp(logit[j] - m);
        sum += pw[j];
      }
      for (int64_t j = 0; j < N; ++j) pw[j] /= sum;
      if (probs)
        for (int64_t j = 0; j < N; ++j) probs[((li * heads + h) * N + i) * N + j] = pw[j];
      double* o = &out[(li * N + i) * C + h * head_dim];
      for (int64_t d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int64_t j = 0; j < N; ++j)
          if (pw[j] != 0.0) acc += pw[j] * widen(v, in_kind, t[j] * token_stride + h * head_dim + d);
        o[d] = acc;
      }
    }
  }
  return 0;
}

// Brute force: dense attention over all real tokens of a sample with an explicit pair
// mask, built in the forward direction from the original coordinate p (a different
// route from orc_window_attn, which maps window slots back to sources):
//   p' = (p - s) mod P per axis, window = p' div w;
//   two tokens of one window are in one pre-shift region iff, on every axis, both or
//   neither lie in the wrapped-around strip p < s (the strip the cyclic shift carried
//   across the seam).
// out : [B][T][H][W][heads*head_dim] doubles.  O(L^2) per sample: tiny grids only.
int orc_dense_masked_attn(const void* q, const void* k, const void* v, int in_kind, int B, int T,
                          int H, int W, int wt, int wh, int ww, int st, int sh, int sw, int heads,
                          int head_dim, int64_t token_stride, double scale, double* out) {
  if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || head_dim < 1) return -1;
  if (st < 0 || sh < 0 || sw < 0 || st >= wt || sh >= wh || sw >= ww) return -1;
  const Geometry g = make_geometry(T, H, W, wt, wh, ww, st, sh, sw);
  if (scale <= 0.0) scale = 1.0 / std::sqrt(static_cast<double>(head_dim));
  const int64_t L = static_cast<int64_t>(T) * H * W;
  const int64_t C = static_cast<int64_t>(heads) * head_dim;
  std::vector<int64_t> win(L);
  std::vector<int> strip(L);
  for (int64_t i = 0; i < L; ++i) {
    const int64_t p[3] = {i / (static_cast<int64_t>(H) * W), (i / W) % H, i % W};
    int64_t wid = 0;
    int bits = 0;
    for (int a = 0; a < 3; ++a) {
      const int64_t pprime = ((p[a] - g.s[a]) % g.P[a] + g.P[a]) % g.P[a];
      wid = wid * g.nwin[a] + pprime / g.w[a];
      bits |= (p[a] < g.s[a] ? 1 : 0) << a;
    }
    win[i] = wid;
    strip[i] = bits;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t job = 0; job < static_cast<int64_t>(B) * heads; ++job) {
    const int64_t b = job / heads, h = job % heads;
    std::vector<double> w(L);
    for (int64_t i = 0; i < L; ++i) {
      const int64_t qi = (b * L + i) * token_stride + h * head_dim;
      double m = -INFINITY;
      for (int64_t j = 0; j < L; ++j) {
        if (win[j] != win[i] || strip[j] != strip[i]) {
          w[j] = -INFINITY;
          continue;
        }
        const int64_t kj = (b * L + j) * token_stride + h * head_dim;
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d) dot += widen(q, in_kind, qi + d) * widen(k, in_kind, kj + d);
        w[j] = scale * dot;
        if (w[j] > m) m = w[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        w[j] = (w[j] == -INFINITY) ? 0.0 : std::exp(w[j] - m);
        sum += w[j];
      }
      double* o = &out[(b * L + i) * C + h * head_dim];
      for (int64_t d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int64_t j = 0; j < L; ++j)
          if (w[j] != 0.0) acc += w[j] * widen(v, in_kind, (b * L + j) * token_stride + h * head_dim + d);
        o[d] = acc / sum;
      }
    }
  }
  return 0;
}

// Fused AdaLN + residual [FA-fusion]: per (sample b, token), over the C channels,
//   mean = sum(x)/C, var = sum((x - mean)^2)/C            (two passes, biased)
//   out  = residual + (x - mean)/sqrt(var + eps) * (1 + scale[b]) + shift[b]
// film_form 0 is the form above; film_form 1 multiplies by scale[b] instead of
// (1 + scale[b]).
// x: [B][L][C] (kind x_kind); residual: [B][L][C] f32 (or null for zero);
// scale, shift: [B][C] f32; out: [B][L][C] doubles.
int orc_adaln(const void* x, int x_kind, const float* residual, const float* scale,
              const float* shift, int B, int64_t L, int C, double eps, int film_form, double* out) {
  if (B < 1 || L < 0 || C < 1 || eps < 0.0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < static_cast<int64_t>(B) * L; ++row) {
    const int64_t b = row / (L > 0 ? L : 1);
    const int64_t base = row * C;
    double mean = 0.0;
    for (int c = 0; c < C; ++c) mean += widen(x, x_kind, base + c);
    mean /= C;
    double var = 0.0;
    for (int c = 0; c < C; ++c) {
      const double d = widen(x, x_kind, base + c) - mean;
      var += d * d;
    }
    var /= C;
    const double inv = 1.0 / std::sqrt(var + eps);
    for (int c = 0; c < C; ++c) {
      const double y = (widen(x, x_kind, base + c) - mean) * inv;
      const double sc = static_cast<double>(scale[b * C + c]);
      const double gain = film_form == 0 ? 1.0 + sc : sc;
      const double res = residual ? static_cast<double>(residual[base + c]) : 0.0;
      out[base + c] = res + y * gain + static_cast<double>(shift[b * C + c]);
    }
  }
  return 0;
}

}  // extern "C"
