// Steps a3 + a4 in fp32 (fp32 operands, fp32 accumulation on the FMA pipe):
// bilinear 4x upsample (align_corners=False) fused into the 1x1 dynamic-kernel
// contraction (the head upsamples the features 4x bilinearly and applies the
// prompts as 1x1 convolution kernels, GKD_GGUF model card, Model section,
// Architecture bullet). Used when the kernel rows are fp32;
// the tensor cores' fp32-input mode (tf32) would not meet a 1e-5 relative bound.
//
// One CTA per (crop, 4x32-pixel tile, group of up to 32 valid rows), 512
// threads: 4 channel quarters x 128 pixels. A thread owns one pixel and every
// fourth 32-channel chunk: it forms the pixel's upsampled slice of the chunk in
// registers (4-tap, dyadic weights) and contracts it against the chunk's rows
// staged in shared memory. The four partial sums of a pixel are added in
// quarter order through shared memory at the end (a fixed order: the result
// does not depend on scheduling).
//
// Decode mode (`keys` non-null): a group holds 16 prompt rows with both
// modality slots side by side, so each thread fuses its pixel's two heatmap
// values in fp32 and the CTA merges one peak key per row into `keys` with
// atomicMax (decode_key.cuh); no heatmap is written.
#include "decode_key.cuh"
#include "gkd_internal.h"

namespace gkd {

constexpr int kF32Pix = 128;                       // pixels per CTA (4 x 32 tile)
constexpr int kF32Quarters = 4;                    // channel quarters per CTA
constexpr int kF32Threads = kF32Pix * kF32Quarters;
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
    const uint8_t* __restrict__ mask, long long mask_bs, int M, int K, float* __restrict__ heat,
    unsigned long long* __restrict__ keys) {
  __shared__ int rows[256];
  __shared__ int krow[128];
  __shared__ int s_nrows;
  extern __shared__ float4 f32_smem[];
  // one row chunk per quarter, then the partial sums of quarters 1..3
  float4 (*ks)[kF32Rows][kF32Chunk / 4] = reinterpret_cast<float4 (*)[kF32Rows][kF32Chunk / 4]>(f32_smem);
  float (*red)[kF32Rows][kF32Pix] =
      reinterpret_cast<float (*)[kF32Rows][kF32Pix]>(f32_smem + kF32Quarters * kF32Rows * (kF32Chunk / 4));

  const int b = blockIdx.z, rg = blockIdx.y;
  const int H = 4 * h, W = 4 * w;
  const int ncb = (W + 31) / 32;
  const int band = blockIdx.x / ncb, cb = blockIdx.x % ncb;
  const uint8_t* mb = mask + static_cast<long long>(b) * mask_bs;
  const bool decode = keys != nullptr;
  if (threadIdx.x == 0) {
    int n = 0;
    if (!decode) {
      for (int r = 0; r < M * K; ++r)
        if (mb[r]) rows[n++] = r;
    } else {
      // slots 2i, 2i+1: modality 0 and 1 of the i-th prompt row with any modality present (-1: absent)
      int nk = 0;
      for (int k = 0; k < K; ++k) {
        const bool p0 = mb[k] != 0, p1 = M == 2 && mb[K + k] != 0;
        if (!p0 && !p1) continue;
        krow[nk] = k;
        rows[2 * nk] = p0 ? k : -1;
        rows[2 * nk + 1] = p1 ? K + k : -1;
        ++nk;
      }
      n = 2 * nk;
    }
    s_nrows = n;
  }
  __syncthreads();
  const int r0 = rg * kF32Rows;
  if (r0 >= s_nrows) return;
  const int nr = min(kF32Rows, s_nrows - r0);

  const int px = threadIdx.x % kF32Pix, qc = threadIdx.x / kF32Pix;   // pixel, channel quarter
  const int Y = 4 * band + (px >> 5);
  const int X = 32 * cb + (px & 31);
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

  const int nchunk = (C + kF32Chunk - 1) / kF32Chunk;
  const int nround = (nchunk + kF32Quarters - 1) / kF32Quarters;
  for (int rd = 0; rd < nround; ++rd) {
    const int c0 = (rd * kF32Quarters + qc) * kF32Chunk;   // this quarter's chunk (may be past C)
    // stage the row chunk: nr rows x 32 channels, by the quarter's 128 threads
    for (int t = px; t < kF32Rows * (kF32Chunk / 4); t += kF32Pix) {
      const int r = t / (kF32Chunk / 4), q = t % (kF32Chunk / 4);
      const int c = c0 + 4 * q;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nr && c < C && rows[r0 + r] >= 0)
        v = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(rows[r0 + r]) * C + c));
      ks[qc][r][q] = v;
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
          const float4 kv = ks[qc][r][q];
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
  // quarter 0 adds the other quarters' partial sums, in quarter order
  if (qc > 0) {
#pragma unroll
    for (int r = 0; r < kF32Rows; ++r)
      if (r < nr) red[qc - 1][r][px] = acc[r];
  }
  __syncthreads();
  if (qc > 0) return;
#pragma unroll
  for (int r = 0; r < kF32Rows; ++r)
    if (r < nr) acc[r] = (acc[r] + red[0][r][px]) + (red[1][r][px] + red[2][r][px]);

  if (decode) {
    // fuse the two modality slots of each prompt row, then one key per row and warp
    const bool inside = Y < H && X < W;
    const uint32_t pixel = inside ? static_cast<uint32_t>(Y * W + X) : 0u;
    const int lane = threadIdx.x & 31;
    unsigned long long mine = 0;
#pragma unroll
    for (int i = 0; i < kF32Rows / 2; ++i) {
      if (2 * i < nr) {
        const bool p0 = rows[r0 + 2 * i] >= 0, p1 = rows[r0 + 2 * i + 1] >= 0;
        const float f = (p0 && p1) ? __fmul_rn(__fadd_rn(acc[2 * i], acc[2 * i + 1]), 0.5f)
                                   : (p0 ? acc[2 * i] : acc[2 * i + 1]);
        uint32_t hi, lo;
        peak_key(f, pixel, inside, hi, lo);
        const unsigned long long key = warp_max_key(hi, lo);
        if (lane == i) mine = key;
      }
    }
    if (mine != 0) atomicMax(keys + static_cast<long long>(b) * K + krow[r0 / 2 + lane], mine);
    return;
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
                               int K, float* heat, unsigned long long* keys, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const int W = 4 * w;
  const int groups = keys ? (K + kF32Rows / 2 - 1) / (kF32Rows / 2) : (M * K + kF32Rows - 1) / kF32Rows;
  dim3 grid(h * ((W + 31) / 32), groups, B);
  const size_t smem = sizeof(float4) * kF32Quarters * kF32Rows * (kF32Chunk / 4) +
                      sizeof(float) * (kF32Quarters - 1) * kF32Rows * kF32Pix;
  cudaError_t e = cudaFuncSetAttribute(heatmap_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  heatmap_f32_kernel<<<grid, kF32Threads, smem, stream>>>(feat, h, w, C, kern, kern_batch_stride, mask,
                                                        mask_batch_stride, M, K, heat, keys);
  return cudaGetLastError();
}

}  // namespace gkd
