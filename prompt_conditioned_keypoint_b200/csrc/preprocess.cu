// The steps on either side of the head, in the ROI geometry of the model card
// (GKD_GGUF, Model section, Input bullet: the ROI's longer side is resized to
// 384 pixels, the result centre-padded to 384 x 384 with the mean colour
// (124, 116, 104) and normalised with the ImageNet mean and standard deviation;
// Output bullet: keypoints come out in the ROI's -1..1 space).
//
// Geometry of a box (x0, y0, x1, y1), canvas side n: s = n / max(bw, bh), pad
// offsets ox = (n - bw s) / 2, oy = (n - bh s) / 2 (not rounded).
//   preprocess: canvas pixel (X, Y) is content iff its centre (X + 0.5, Y + 0.5)
//     lies in [ox, ox + bw s) x [oy, oy + bh s); content takes the bilinear
//     sample of the image at x0 + (X + 0.5 - ox) / s - 0.5 (and likewise y),
//     taps clamped to the image; the rest takes the pad colour; then
//     (v / 255 - mean) / std per channel, channel-major output.
//   ROI -> image: u in -1..1 -> canvas pixel (u + 1) n / 2 -> x0 + (p - ox) / s.
// Arithmetic in fp64 with every operation rounded separately, in the order the
// formulas are written (no contraction), and one rounding to fp32 at the end.
#include <cmath>

#include "gkd_internal.h"

namespace gkd {

struct BoxGeom {
  double x0, y0, s, ox, oy, bw, bh;
  bool ok;
};

__device__ __forceinline__ BoxGeom box_geom(const float* box, int canvas) {
  BoxGeom g;
  g.x0 = box[0];
  g.y0 = box[1];
  g.bw = __dsub_rn(static_cast<double>(box[2]), g.x0);
  g.bh = __dsub_rn(static_cast<double>(box[3]), g.y0);
  g.ok = g.bw > 0.0 && g.bh > 0.0 && isfinite(g.bw) && isfinite(g.bh) && isfinite(g.x0) && isfinite(g.y0);
  const double n = static_cast<double>(canvas);
  g.s = __ddiv_rn(n, fmax(g.bw, g.bh));
  g.ox = __ddiv_rn(__dsub_rn(n, __dmul_rn(g.bw, g.s)), 2.0);
  g.oy = __ddiv_rn(__dsub_rn(n, __dmul_rn(g.bh, g.s)), 2.0);
  return g;
}

struct AxisTap {
  int i0, i1;
  double lam;
  bool inside;
};

__device__ __forceinline__ AxisTap axis_tap(int d, int n_in, double origin, double s, double off, double extent) {
  AxisTap t;
  const double c = __dadd_rn(static_cast<double>(d), 0.5);
  t.inside = c >= off && c < __dadd_rn(off, __dmul_rn(s, extent));
  const double x = __dsub_rn(__dadd_rn(origin, __ddiv_rn(__dsub_rn(c, off), s)), 0.5);
  const double f = floor(x);
  t.lam = __dsub_rn(x, f);
  const double hi = static_cast<double>(n_in - 1);
  t.i0 = static_cast<int>(fmin(fmax(f, 0.0), hi));
  t.i1 = static_cast<int>(fmin(fmax(__dadd_rn(f, 1.0), 0.0), hi));
  return t;
}

__device__ __forceinline__ float normalise(double v, int c) {
  const double mean[3] = {0.485, 0.456, 0.406};
  const double stdv[3] = {0.229, 0.224, 0.225};
  return static_cast<float>(__ddiv_rn(__dsub_rn(__ddiv_rn(v, 255.0), mean[c]), stdv[c]));
}

// One CTA per (box, band of kPpRows canvas rows). Every value is computed as
// the per-pixel formulas state; what depends on one axis only is computed once
// and reused: the box geometry per thread, the row taps per band (shared
// memory), a column's taps once for the band's rows, and the normalised pad
// colour once per thread.
constexpr int kPpRows = 8;

__global__ void __launch_bounds__(256) preprocess_kernel(const uint8_t* __restrict__ img, int H, int W,
                                                         const float* __restrict__ boxes, int canvas,
                                                         float* __restrict__ out) {
  __shared__ AxisTap rowtap[kPpRows];
  const int b = blockIdx.y;
  const int Y0 = blockIdx.x * kPpRows;
  const int nr = min(kPpRows, canvas - Y0);
  const long long npx = static_cast<long long>(canvas) * canvas;
  const BoxGeom g = box_geom(boxes + 4 * static_cast<long long>(b), canvas);
  if (g.ok && threadIdx.x < nr) rowtap[threadIdx.x] = axis_tap(Y0 + threadIdx.x, H, g.y0, g.s, g.oy, g.bh);
  __syncthreads();
  const float padn[3] = {normalise(124.0, 0), normalise(116.0, 1), normalise(104.0, 2)};
  float* ob = out + static_cast<long long>(b) * 3 * npx + static_cast<long long>(Y0) * canvas;
  for (int X = threadIdx.x; X < canvas; X += blockDim.x) {
    AxisTap tx{};
    if (g.ok) tx = axis_tap(X, W, g.x0, g.s, g.ox, g.bw);
    const double wx0 = __dsub_rn(1.0, tx.lam);
    for (int r = 0; r < nr; ++r) {
      float o[3] = {padn[0], padn[1], padn[2]};
      if (g.ok && tx.inside && rowtap[r].inside) {
        const AxisTap ty = rowtap[r];
        const uint8_t* r0 = img + static_cast<long long>(ty.i0) * W * 3;
        const uint8_t* r1 = img + static_cast<long long>(ty.i1) * W * 3;
        const double wy0 = __dsub_rn(1.0, ty.lam);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const double a = r0[3 * tx.i0 + c], bb = r0[3 * tx.i1 + c];
          const double cc = r1[3 * tx.i0 + c], d = r1[3 * tx.i1 + c];
          const double top = __dadd_rn(__dmul_rn(wx0, a), __dmul_rn(tx.lam, bb));
          const double bot = __dadd_rn(__dmul_rn(wx0, cc), __dmul_rn(tx.lam, d));
          o[c] = normalise(__dadd_rn(__dmul_rn(wy0, top), __dmul_rn(ty.lam, bot)), c);
        }
      }
      const long long q = static_cast<long long>(r) * canvas + X;
#pragma unroll
      for (int c = 0; c < 3; ++c) ob[c * npx + q] = o[c];
    }
  }
}

__global__ void __launch_bounds__(256) roi_to_image_kernel(const float* __restrict__ xy,
                                                           const float* __restrict__ boxes, int B, int K,
                                                           int canvas, float* __restrict__ out) {
  const long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (o >= static_cast<long long>(B) * K) return;
  const int b = static_cast<int>(o / K);
  const BoxGeom g = box_geom(boxes + 4 * static_cast<long long>(b), canvas);
  if (!g.ok) {
    out[2 * o] = out[2 * o + 1] = __int_as_float(0x7FC00000);
    return;
  }
  const double n = static_cast<double>(canvas);
  const double px = __ddiv_rn(__dmul_rn(__dadd_rn(static_cast<double>(xy[2 * o]), 1.0), n), 2.0);
  const double py = __ddiv_rn(__dmul_rn(__dadd_rn(static_cast<double>(xy[2 * o + 1]), 1.0), n), 2.0);
  out[2 * o] = static_cast<float>(__dadd_rn(g.x0, __ddiv_rn(__dsub_rn(px, g.ox), g.s)));
  out[2 * o + 1] = static_cast<float>(__dadd_rn(g.y0, __ddiv_rn(__dsub_rn(py, g.oy), g.s)));
}

cudaError_t launch_preprocess(const uint8_t* img, int H, int W, const float* boxes, int B, int canvas, float* out,
                              cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((canvas + kPpRows - 1) / kPpRows), B);
  preprocess_kernel<<<grid, 256, 0, stream>>>(img, H, W, boxes, canvas, out);
  return cudaGetLastError();
}

cudaError_t launch_roi_to_image(const float* xy, const float* boxes, int B, int K, int canvas, float* out,
                                cudaStream_t stream) {
  const long long n = static_cast<long long>(B) * K;
  if (n == 0) return cudaSuccess;
  roi_to_image_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(xy, boxes, B, K, canvas, out);
  return cudaGetLastError();
}

}  // namespace gkd
