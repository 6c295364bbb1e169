// Steps a3 + a4 in fp32 (fp32 operands, fp32 accumulation on the FMA pipe):
// bilinear 4x upsample (align_corners=False) fused into the 1x1 dynamic-kernel
// contraction (the head upsamples the features 4x bilinearly and applies the
// prompts as 1x1 convolution kernels, GKD_GGUF model card, Model section,
// Architecture bullet). Used when the kernel rows are fp32;
// the tensor cores' fp32-input mode (tf32) would not meet a 1e-5 relative bound.
//
// One CTA per (crop, 4x32-pixel tile, group of up to 32 valid rows): each
// thread owns one pixel, forms its upsampled 32-channel slice in registers
// (4-tap, dyadic weights) and contracts it against the row chunk staged in
// shared memory.
#include "gkd_internal.h"

namespace gkd {

constexpr int kF32Threads = 128;
constexpr int kF32Rows = 32;
constexpr int kF32Chunk = 32;

__device__ __forceinline__ void taps_f32(int d, int n, int& i0, int& i1, float& lam) {
  const float s = fmaxf((static_cast<float>(d) + 0.5f) * 0.25f - 0.5f, 0.0f);
  i0 = min(static_cast<int>(s), n - 1);
  i1 = min(i0 + 1, n - 1);
  lam = s - static_cast<float>(static_cast<int>(s));
}

__global__ void __launch_bounds__(kF32Threads) heatmap_f32_kernel(
    const float* __restrict__ feat, int h, int w, int C, const float* __restrict__ kern, long long kern_bs,
    const uint8_t* __restrict__ mask, long long mask_bs, int M, int K, float* __restrict__ heat) {
  __shared__ int rows[256];
  __shared__ int s_nrows;
  __shared__ float4 ks[kF32Rows][kF32Chunk / 4];

  const int b = blockIdx.z, rg = blockIdx.y;
  const int H = 4 * h, W = 4 * w;
  const int ncb = (W + 31) / 32;
  const int band = blockIdx.x / ncb, cb = blockIdx.x % ncb;
  const uint8_t* mb = mask + static_cast<long long>(b) * mask_bs;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int r = 0; r < M * K; ++r)
      if (mb[r]) rows[n++] = r;
    s_nrows = n;
  }
  __syncthreads();
  const int r0 = rg * kF32Rows;
  if (r0 >= s_nrows) return;
  const int nr = min(kF32Rows, s_nrows - r0);

  const int Y = 4 * band + (threadIdx.x >> 5);
  const int X = 32 * cb + (threadIdx.x & 31);
  int y0, y1, x0, x1;
  float ly, lx;
  taps_f32(Y, h, y0, y1, ly);
  taps_f32(min(X, W - 1), w, x0, x1, lx);
  const float w00 = (1.f - ly) * (1.f - lx), w01 = (1.f - ly) * lx, w10 = ly * (1.f - lx), w11 = ly * lx;
  const float* Fb = feat + static_cast<long long>(b) * h * w * C;
  const float* p00 = Fb + (static_cast<long long>(y0) * w + x0) * C;
  const float* p01 = Fb + (static_cast<long long>(y0) * w + x1) * C;
  const float* p10 = Fb + (static_cast<long long>(y1) * w + x0) * C;
  const float* p11 = Fb + (static_cast<long long>(y1) * w + x1) * C;
  const float* kb = kern + static_cast<long long>(b) * kern_bs;

  float acc[kF32Rows];
#pragma unroll
  for (int r = 0; r < kF32Rows; ++r) acc[r] = 0.f;

  for (int c0 = 0; c0 < C; c0 += kF32Chunk) {
    // stage the row chunk: nr rows x 32 channels
    for (int t = threadIdx.x; t < kF32Rows * (kF32Chunk / 4); t += blockDim.x) {
      const int r = t / (kF32Chunk / 4), q = t % (kF32Chunk / 4);
      const int c = c0 + 4 * q;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nr && c < C) v = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(rows[r0 + r]) * C + c));
      ks[r][q] = v;
    }
    // this pixel's upsampled channels
    float u[kF32Chunk];
#pragma unroll
    for (int q = 0; q < kF32Chunk / 4; ++q) {
      const int c = c0 + 4 * q;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bq = a, cq = a, dq = a;
      if (c < C) {
        a = __ldg(reinterpret_cast<const float4*>(p00 + c));
        bq = __ldg(reinterpret_cast<const float4*>(p01 + c));
        cq = __ldg(reinterpret_cast<const float4*>(p10 + c));
        dq = __ldg(reinterpret_cast<const float4*>(p11 + c));
      }
      u[4 * q + 0] = fmaf(w11, dq.x, fmaf(w10, cq.x, fmaf(w01, bq.x, w00 * a.x)));
      u[4 * q + 1] = fmaf(w11, dq.y, fmaf(w10, cq.y, fmaf(w01, bq.y, w00 * a.y)));
      u[4 * q + 2] = fmaf(w11, dq.z, fmaf(w10, cq.z, fmaf(w01, bq.z, w00 * a.z)));
      u[4 * q + 3] = fmaf(w11, dq.w, fmaf(w10, cq.w, fmaf(w01, bq.w, w00 * a.w)));
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kF32Rows; ++r) {
      if (r < nr) {
        float s = acc[r];
#pragma unroll
        for (int q = 0; q < kF32Chunk / 4; ++q) {
          const float4 kv = ks[r][q];
          s = fmaf(u[4 * q + 0], kv.x, s);
          s = fmaf(u[4 * q + 1], kv.y, s);
          s = fmaf(u[4 * q + 2], kv.z, s);
          s = fmaf(u[4 * q + 3], kv.w, s);
        }
        acc[r] = s;
      }
    }
    __syncthreads();
  }

  if (Y < H && X < W) {
    const long long P = static_cast<long long>(H) * W;
    float* hb = heat + static_cast<long long>(b) * M * K * P + static_cast<long long>(Y) * W + X;
#pragma unroll
    for (int r = 0; r < kF32Rows; ++r)
      if (r < nr) hb[static_cast<long long>(rows[r0 + r]) * P] = acc[r];
  }
}

cudaError_t launch_heatmap_f32(const float* feat, int B, int h, int w, int C, const float* kern,
                               long long kern_batch_stride, const uint8_t* mask, long long mask_batch_stride, int M,
                               int K, float* heat, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const int W = 4 * w;
  dim3 grid(h * ((W + 31) / 32), (M * K + kF32Rows - 1) / kF32Rows, B);
  heatmap_f32_kernel<<<grid, kF32Threads, 0, stream>>>(feat, h, w, C, kern, kern_batch_stride, mask,
                                                        mask_batch_stride, M, K, heat);
  return cudaGetLastError();
}

}  // namespace gkd
