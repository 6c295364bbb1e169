// Step a1: Gaussian prototype pooling of support-image patch features at the
// annotated keypoints. Visual prompts are one-shot keypoints pooled with a
// Gaussian of sigma 14 px (GKD_GGUF model card, Model section, Prompts bullet);
// the prototypes come from Gaussian weights placed on the support image at the
// keypoints (GKDT summary page, pipeline paragraph).
//
// proto[b,k,:] = sum_ij w_ij F[b,i,j,:] / sum_ij w_ij with
// w_ij = exp(-((X_j - x)^2 + (Y_i - y)^2) / (2 sigma^2)) at patch centres
// X_j = stride (j + 0.5), Y_i = stride (i + 0.5). The weight separates into
// gx[j] * gy[i]; each factor is divided by its largest value (a common factor
// that cancels in the ratio), so the denominator never underflows.
//
// One CTA per (crop, 128-channel block): 32 lanes x 4 channels (128-bit loads)
// and 8 keypoint groups; the per-keypoint factors live in shared memory.
#include "gkd_internal.h"

namespace gkd {

constexpr int kPoolThreads = 256;
constexpr int kPoolGroups = kPoolThreads / 32;     // keypoint groups
constexpr int kPoolMaxPerThread = 16;              // K <= 128

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(
    const float* __restrict__ support, int h, int w, int C, const float* __restrict__ kpts,
    const uint8_t* __restrict__ kmask, int K, float sigma, float stride, float* __restrict__ proto,
    long long proto_bs) {
  extern __shared__ float sm[];
  int* klist = reinterpret_cast<int*>(sm);           // [K]
  float* inv = sm + K;                               // [K]
  float* gx = inv + K;                               // [K][w]
  float* gy = gx + K * w;                            // [K][h]
  __shared__ int s_nv;

  const int b = blockIdx.y;
  const int c0 = blockIdx.x * 128;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const uint8_t* km = kmask + static_cast<long long>(b) * K;
  const float* kp = kpts + static_cast<long long>(b) * K * 2;

  if (threadIdx.x == 0) {
    int n = 0;
    for (int k = 0; k < K; ++k)
      if (km[k]) klist[n++] = k;
    s_nv = n;
  }
  __syncthreads();
  const int nv = s_nv;

  // squared distances to the patch centres
  for (int t = threadIdx.x; t < nv * w; t += blockDim.x) {
    const int kk = t / w, j = t - kk * w;
    const float d = stride * (static_cast<float>(j) + 0.5f) - kp[2 * klist[kk]];
    gx[t] = d * d;
  }
  for (int t = threadIdx.x; t < nv * h; t += blockDim.x) {
    const int kk = t / h, i = t - kk * h;
    const float d = stride * (static_cast<float>(i) + 0.5f) - kp[2 * klist[kk] + 1];
    gy[t] = d * d;
  }
  __syncthreads();

  // factors exp(-(d2 - d2min) / (2 sigma^2)) and the normaliser, one warp per keypoint
  const float inv2s2 = 1.0f / (2.0f * sigma * sigma);
  for (int kk = ty; kk < nv; kk += kPoolGroups) {
    float* fx = gx + kk * w;
    float* fy = gy + kk * h;
    float mx = INFINITY, my = INFINITY;
    for (int j = tx; j < w; j += 32) mx = fminf(mx, fx[j]);
    for (int i = tx; i < h; i += 32) my = fminf(my, fy[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fminf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      my = fminf(my, __shfl_xor_sync(0xffffffffu, my, o));
    }
    float sx = 0.f, sy = 0.f;
    for (int j = tx; j < w; j += 32) {
      const float e = expf(-(fx[j] - mx) * inv2s2);
      fx[j] = e;
      sx += e;
    }
    for (int i = tx; i < h; i += 32) {
      const float e = expf(-(fy[i] - my) * inv2s2);
      fy[i] = e;
      sy += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, o);
      sy += __shfl_xor_sync(0xffffffffu, sy, o);
    }
    if (tx == 0) inv[kk] = 1.0f / (sx * sy);
  }
  __syncthreads();

  const int c = c0 + 4 * tx;
  const bool cok = c < C;
  float4 acc[kPoolMaxPerThread];
#pragma unroll
  for (int t = 0; t < kPoolMaxPerThread; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);

  const float* Fb = support + static_cast<long long>(b) * h * w * C;
  for (int i = 0; i < h; ++i) {
    float wy[kPoolMaxPerThread];
#pragma unroll
    for (int t = 0; t < kPoolMaxPerThread; ++t) {
      const int kk = ty + kPoolGroups * t;
      wy[t] = (kk < nv) ? gy[kk * h + i] : 0.f;
    }
    const float* Frow = Fb + static_cast<long long>(i) * w * C;
    for (int j = 0; j < w; ++j) {
      const float4 f = cok ? __ldg(reinterpret_cast<const float4*>(Frow + static_cast<long long>(j) * C + c))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int t = 0; t < kPoolMaxPerThread; ++t) {
        const int kk = ty + kPoolGroups * t;
        if (kk < nv) {
          const float wv = wy[t] * gx[kk * w + j];
          acc[t].x = fmaf(wv, f.x, acc[t].x);
          acc[t].y = fmaf(wv, f.y, acc[t].y);
          acc[t].z = fmaf(wv, f.z, acc[t].z);
          acc[t].w = fmaf(wv, f.w, acc[t].w);
        }
      }
    }
  }

  float* Pb = proto + static_cast<long long>(b) * proto_bs;
  if (cok) {
#pragma unroll
    for (int t = 0; t < kPoolMaxPerThread; ++t) {
      const int kk = ty + kPoolGroups * t;
      if (kk < nv) {
        const float s = inv[kk];
        const float4 r = make_float4(acc[t].x * s, acc[t].y * s, acc[t].z * s, acc[t].w * s);
        *reinterpret_cast<float4*>(Pb + static_cast<long long>(klist[kk]) * C + c) = r;
      }
    }
    // invalid keypoints get zero rows
    for (int k = ty; k < K; k += kPoolGroups)
      if (!km[k]) *reinterpret_cast<float4*>(Pb + static_cast<long long>(k) * C + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

size_t pool_smem_bytes(int h, int w, int K) {
  return sizeof(float) * (2 * static_cast<size_t>(K) + static_cast<size_t>(K) * (w + h));
}

cudaError_t launch_pool(const float* support, int B, int h, int w, int C, const float* kpts,
                        const uint8_t* kmask, int K, float sigma, float stride, float* proto,
                        long long proto_batch_stride, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const size_t smem = pool_smem_bytes(h, w, K);
  cudaError_t e = cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((C + 127) / 128, B);
  pool_kernel<<<grid, kPoolThreads, smem, stream>>>(support, h, w, C, kpts, kmask, K, sigma, stride, proto,
                                                     proto_batch_stride);
  return cudaGetLastError();
}

}  // namespace gkd
