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
// One CTA per (128-channel block, crop, slice of 16 keypoints): the 8 warps
// split the source rows (row i goes to warp i % 8), each thread accumulates 4
// channels x the slice's valid keypoints over its warp's rows, and the 8 partial
// sums are added in a fixed order through shared memory at the end (the result
// does not depend on scheduling). Enough CTAs to fill the SMs even for one crop,
// and each warp keeps a float4 load per pixel in flight against 16 keypoints' FMAs.
#include "gkd_internal.h"

namespace gkd {

constexpr int kPoolThreads = 256;
constexpr int kPoolWarps = kPoolThreads / 32;
constexpr int kPoolSlice = 16;                     // keypoints per CTA

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(
    const float* __restrict__ support, int h, int w, int C, const float* __restrict__ kpts,
    const uint8_t* __restrict__ kmask, int K, float sigma, float stride, float* __restrict__ proto,
    long long proto_bs) {
  extern __shared__ float sm[];
  float* gx = sm;                                    // [kPoolSlice][w]
  float* gy = gx + kPoolSlice * w;                   // [kPoolSlice][h]
  float4* red = reinterpret_cast<float4*>(gy + kPoolSlice * h + ((4 - (kPoolSlice * (w + h)) % 4) % 4));
                                                     // [kPoolWarps][kPoolSlice][32] float4
  __shared__ int klist[kPoolSlice];
  __shared__ float inv[kPoolSlice];
  __shared__ int s_nv;

  const int cb = blockIdx.x, b = blockIdx.y, k0 = blockIdx.z * kPoolSlice;
  const int c0 = cb * 128;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint8_t* km = kmask + static_cast<long long>(b) * K;
  const float* kp = kpts + static_cast<long long>(b) * K * 2;
  const int kend = min(K, k0 + kPoolSlice);

  if (threadIdx.x == 0) {
    int n = 0;
    for (int k = k0; k < kend; ++k)
      if (km[k]) klist[n++] = k;
    s_nv = n;
  }
  __syncthreads();
  const int nv = s_nv;
  const int c = c0 + 4 * lane;
  const bool cok = c < C;
  float* Pb = proto + static_cast<long long>(b) * proto_bs;
  // absent keypoints of the slice get zero rows
  if (cok)
    for (int k = k0 + warp; k < kend; k += kPoolWarps)
      if (!km[k]) *reinterpret_cast<float4*>(Pb + static_cast<long long>(k) * C + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  if (nv == 0) return;

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
  for (int kk = warp; kk < nv; kk += kPoolWarps) {
    float* fx = gx + kk * w;
    float* fy = gy + kk * h;
    float mx = INFINITY, my = INFINITY;
    for (int j = lane; j < w; j += 32) mx = fminf(mx, fx[j]);
    for (int i = lane; i < h; i += 32) my = fminf(my, fy[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fminf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      my = fminf(my, __shfl_xor_sync(0xffffffffu, my, o));
    }
    float sx = 0.f, sy = 0.f;
    for (int j = lane; j < w; j += 32) {
      const float e = expf(-(fx[j] - mx) * inv2s2);
      fx[j] = e;
      sx += e;
    }
    for (int i = lane; i < h; i += 32) {
      const float e = expf(-(fy[i] - my) * inv2s2);
      fy[i] = e;
      sy += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, o);
      sy += __shfl_xor_sync(0xffffffffu, sy, o);
    }
    if (lane == 0) inv[kk] = 1.0f / (sx * sy);
  }
  __syncthreads();

  float4 acc[kPoolSlice];
#pragma unroll
  for (int t = 0; t < kPoolSlice; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);

  const float* Fb = support + static_cast<long long>(b) * h * w * C;
  for (int i = warp; i < h; i += kPoolWarps) {
    float wy[kPoolSlice];
#pragma unroll
    for (int t = 0; t < kPoolSlice; ++t) wy[t] = (t < nv) ? gy[t * h + i] : 0.f;
    const float* Frow = Fb + static_cast<long long>(i) * w * C + c;
    int j = 0;
    for (; j + 4 <= w; j += 4) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        f[u] = cok ? __ldg(reinterpret_cast<const float4*>(Frow + static_cast<long long>(j + u) * C))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int t = 0; t < kPoolSlice; ++t) {
          if (t < nv) {
            const float wv = wy[t] * gx[t * w + j + u];
            acc[t].x = fmaf(wv, f[u].x, acc[t].x);
            acc[t].y = fmaf(wv, f[u].y, acc[t].y);
            acc[t].z = fmaf(wv, f[u].z, acc[t].z);
            acc[t].w = fmaf(wv, f[u].w, acc[t].w);
          }
        }
      }
    }
    for (; j < w; ++j) {
      const float4 f = cok ? __ldg(reinterpret_cast<const float4*>(Frow + static_cast<long long>(j) * C))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int t = 0; t < kPoolSlice; ++t) {
        if (t < nv) {
          const float wv = wy[t] * gx[t * w + j];
          acc[t].x = fmaf(wv, f.x, acc[t].x);
          acc[t].y = fmaf(wv, f.y, acc[t].y);
          acc[t].z = fmaf(wv, f.z, acc[t].z);
          acc[t].w = fmaf(wv, f.w, acc[t].w);
        }
      }
    }
  }

  // partial sums of the 8 warps, added in warp order
#pragma unroll
  for (int t = 0; t < kPoolSlice; ++t)
    if (t < nv) red[(warp * kPoolSlice + t) * 32 + lane] = acc[t];
  __syncthreads();
  for (int o = threadIdx.x; o < nv * 32; o += blockDim.x) {
    const int t = o >> 5, l = o & 31;
    const int cc = c0 + 4 * l;
    if (cc >= C) continue;
    float4 sum = red[t * 32 + l];
#pragma unroll
    for (int wp = 1; wp < kPoolWarps; ++wp) {
      const float4 v = red[(wp * kPoolSlice + t) * 32 + l];
      sum.x += v.x;
      sum.y += v.y;
      sum.z += v.z;
      sum.w += v.w;
    }
    const float sc = inv[t];
    *reinterpret_cast<float4*>(Pb + static_cast<long long>(klist[t]) * C + cc) =
        make_float4(sum.x * sc, sum.y * sc, sum.z * sc, sum.w * sc);
  }
}

size_t pool_smem_bytes(int h, int w, int K) {
  (void)K;
  const size_t f = static_cast<size_t>(kPoolSlice) * (w + h);
  return sizeof(float) * (f + (4 - f % 4) % 4) + sizeof(float4) * kPoolWarps * kPoolSlice * 32;
}

cudaError_t launch_pool(const float* support, int B, int h, int w, int C, const float* kpts,
                        const uint8_t* kmask, int K, float sigma, float stride, float* proto,
                        long long proto_batch_stride, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const size_t smem = pool_smem_bytes(h, w, K);
  cudaError_t e = cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((C + 127) / 128, B, (K + kPoolSlice - 1) / kPoolSlice);
  pool_kernel<<<grid, kPoolThreads, smem, stream>>>(support, h, w, C, kpts, kmask, K, sigma, stride, proto,
                                                     proto_batch_stride);
  return cudaGetLastError();
}

}  // namespace gkd
