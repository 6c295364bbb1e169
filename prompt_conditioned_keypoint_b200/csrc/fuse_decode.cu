// Steps a5 + a6: per-row masked fusion across prompt modalities (prompt rows are
// padded to 80 and fused row by row under a validity mask, GKD_GGUF model card,
// Model section, Architecture bullet; text and visual prompts may be combined
// row by row, Prompts bullet), then the peak of each fused heatmap mapped to ROI
// coordinates in -1..1 with a confidence score (the output is the per-prompt
// peak on the 96x96 grid in the ROI's normalised space, Output bullet).
//
// fused = H_v or H_t when one modality is present, (H_v + H_t) * 0.5 in fp32 when
// both are; the peak is the first (lowest row-major index) maximal pixel;
// x = (2 col + 1 - W) / W and y = (2 row + 1 - H) / H in one IEEE division each.
// One CTA per (crop, row): 128-bit streaming loads, then a warp-shuffle and
// shared-memory (value, index) reduction.
#include <climits>

#include "gkd_internal.h"

namespace gkd {

constexpr int kDecThreads = 256;

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// UNROLL > 1 (long rows): several iterations' loads are in flight before the
// serial comparisons consume them; the visiting order, and so the result, is
// unchanged. Short rows (workload 2's 9 iterations per thread) run faster
// without it.
template <int UNROLL>
__global__ void __launch_bounds__(kDecThreads) fuse_decode_kernel(
    const float* __restrict__ heat, const uint8_t* __restrict__ mask, long long mask_bs, int M, int K, int H,
    int W, float* __restrict__ fused, float* __restrict__ xy, float* __restrict__ score,
    int32_t* __restrict__ idx, uint8_t* __restrict__ valid) {
  const int k = blockIdx.x, b = blockIdx.y;
  const uint8_t* mb = mask + static_cast<long long>(b) * mask_bs;
  const bool hv = mb[k] != 0;
  const bool ht = (M == 2) && (mb[K + k] != 0);
  const long long o = static_cast<long long>(b) * K + k;
  const int P = H * W;
  float4* frow = fused ? reinterpret_cast<float4*>(fused + o * P) : nullptr;

  if (!hv && !ht) {
    if (threadIdx.x == 0) {
      idx[o] = -1;
      valid[o] = 0;
      score[o] = 0.f;
      xy[2 * o] = 0.f;
      xy[2 * o + 1] = 0.f;
    }
    if (frow)
      for (int p = threadIdx.x; p < P / 4; p += blockDim.x) frow[p] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }

  const float4* rv = reinterpret_cast<const float4*>(heat + (static_cast<long long>(b) * M * K + k) * P);
  const float4* rt = reinterpret_cast<const float4*>(heat + (static_cast<long long>(b) * M * K + K + k) * P);
  float best = -INFINITY;
  int bi = INT_MAX;
#pragma unroll UNROLL
  for (int p = threadIdx.x; p < P / 4; p += blockDim.x) {
    float4 f;
    if (hv && ht) {
      const float4 a = __ldcs(rv + p), c = __ldcs(rt + p);
      f = make_float4(__fmul_rn(__fadd_rn(a.x, c.x), 0.5f), __fmul_rn(__fadd_rn(a.y, c.y), 0.5f),
                      __fmul_rn(__fadd_rn(a.z, c.z), 0.5f), __fmul_rn(__fadd_rn(a.w, c.w), 0.5f));
    } else {
      f = __ldcs(hv ? rv + p : rt + p);
    }
    if (frow) frow[p] = f;
    const int i0 = 4 * p;
    if (better(f.x, i0, best, bi)) { best = f.x; bi = i0; }
    if (better(f.y, i0 + 1, best, bi)) { best = f.y; bi = i0 + 1; }
    if (better(f.z, i0 + 2, best, bi)) { best = f.z; bi = i0 + 2; }
    if (better(f.w, i0 + 3, best, bi)) { best = f.w; bi = i0 + 3; }
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    const float v = __shfl_xor_sync(0xffffffffu, best, s);
    const int i = __shfl_xor_sync(0xffffffffu, bi, s);
    if (better(v, i, best, bi)) { best = v; bi = i; }
  }
  __shared__ float sv[kDecThreads / 32];
  __shared__ int si[kDecThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[warp] = best; si[warp] = bi; }
  __syncthreads();
  if (warp == 0) {
    best = lane < kDecThreads / 32 ? sv[lane] : -INFINITY;
    bi = lane < kDecThreads / 32 ? si[lane] : INT_MAX;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      const float v = __shfl_xor_sync(0xffffffffu, best, s);
      const int i = __shfl_xor_sync(0xffffffffu, bi, s);
      if (better(v, i, best, bi)) { best = v; bi = i; }
    }
    if (lane == 0) {
      if (bi == INT_MAX) {   // no pixel compared (every value NaN): report the first pixel
        bi = 0;
        const float a0 = hv ? reinterpret_cast<const float*>(rv)[0] : 0.f;
        const float c0 = ht ? reinterpret_cast<const float*>(rt)[0] : 0.f;
        best = (hv && ht) ? __fmul_rn(__fadd_rn(a0, c0), 0.5f) : (hv ? a0 : c0);
      }
      const int col = bi % W, row = bi / W;
      idx[o] = bi;
      valid[o] = 1;
      score[o] = best;
      xy[2 * o] = __fdiv_rn(static_cast<float>(2 * col + 1 - W), static_cast<float>(W));
      xy[2 * o + 1] = __fdiv_rn(static_cast<float>(2 * row + 1 - H), static_cast<float>(H));
    }
  }
}

// Decode fused into the heatmap kernels: turn the per-(crop, row) peak keys
// (decode_key.cuh) into the same outputs as fuse_decode_kernel. One thread per
// (crop, row).
__global__ void __launch_bounds__(256) finalize_keys_kernel(const unsigned long long* __restrict__ keys,
                                                            const uint8_t* __restrict__ mask, long long mask_bs,
                                                            int B, int M, int K, int H, int W,
                                                            float* __restrict__ xy, float* __restrict__ score,
                                                            int32_t* __restrict__ idx, uint8_t* __restrict__ valid) {
  const long long o = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (o >= static_cast<long long>(B) * K) return;
  const int b = static_cast<int>(o / K), k = static_cast<int>(o % K);
  const uint8_t* mb = mask + static_cast<long long>(b) * mask_bs;
  const bool present = mb[k] != 0 || (M == 2 && mb[K + k] != 0);
  if (!present) {
    idx[o] = -1;
    valid[o] = 0;
    score[o] = 0.f;
    xy[2 * o] = 0.f;
    xy[2 * o + 1] = 0.f;
    return;
  }
  const unsigned long long key = keys[o];
  int p = 0;
  float v = __uint_as_float(0x7FC00000u);     // no candidate: every value was NaN
  if (key != 0) {
    const uint32_t hi = static_cast<uint32_t>(key >> 32), lo = static_cast<uint32_t>(key);
    p = static_cast<int>(0x7FFFFFFFu - (lo >> 1));
    uint32_t u = (hi & 0x80000000u) ? (hi & 0x7FFFFFFFu) : ~hi;
    if (u == 0 && (lo & 1u)) u = 0x80000000u;    // the peak was -0
    v = __uint_as_float(u);
  }
  const int col = p % W, row = p / W;
  idx[o] = p;
  valid[o] = 1;
  score[o] = v;
  xy[2 * o] = __fdiv_rn(static_cast<float>(2 * col + 1 - W), static_cast<float>(W));
  xy[2 * o + 1] = __fdiv_rn(static_cast<float>(2 * row + 1 - H), static_cast<float>(H));
}

cudaError_t launch_finalize_keys(const unsigned long long* keys, const uint8_t* mask, long long mask_batch_stride,
                                 int B, int M, int K, int H, int W, float* xy, float* score, int32_t* idx,
                                 uint8_t* valid, cudaStream_t stream) {
  const long long n = static_cast<long long>(B) * K;
  if (n == 0) return cudaSuccess;
  finalize_keys_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
      keys, mask, mask_batch_stride, B, M, K, H, W, xy, score, idx, valid);
  return cudaGetLastError();
}

cudaError_t launch_fuse_decode(const float* heat, const uint8_t* mask, long long mask_batch_stride, int B, int M,
                               int K, int H, int W, float* fused, float* xy, float* score, int32_t* idx,
                               uint8_t* valid, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  dim3 grid(K, B);
  if (H * W / 4 >= 16 * kDecThreads)   // 16 or more float4 per thread
    fuse_decode_kernel<4><<<grid, kDecThreads, 0, stream>>>(heat, mask, mask_batch_stride, M, K, H, W, fused, xy,
                                                            score, idx, valid);
  else
    fuse_decode_kernel<1><<<grid, kDecThreads, 0, stream>>>(heat, mask, mask_batch_stride, M, K, H, W, fused, xy,
                                                            score, idx, valid);
  return cudaGetLastError();
}

}  // namespace gkd
