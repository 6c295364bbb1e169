// Step a2: L2 normalisation of prompt rows: the head normalises each kernel row
// to unit L2 norm (GKD_GGUF model card, Model section, Architecture bullet; the
// convolution with prompts is a normalised one, GKDT reading notes, Method
// section). One warp per row: 128-bit loads, fp32 sum of squares, warp-shuffle
// reduction, IEEE sqrt and division, optional round-to-nearest-even bf16 output.
#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {

template <bool OUT_BF16>
__global__ void __launch_bounds__(256) norm_rows_kernel(const float* __restrict__ rows,
                                                        const uint8_t* __restrict__ mask, long long nrows,
                                                        int C, float eps, void* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= nrows) return;
  const float4* src = reinterpret_cast<const float4*>(rows + row * C);
  const int nq = C >> 2;
  const bool valid = mask[row] != 0;
  float ss = 0.f;
  if (valid) {
    for (int i = lane; i < nq; i += 32) {
      const float4 v = __ldg(src + i);
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const float d = fmaxf(__fsqrt_rn(ss), eps);
  if (OUT_BF16) {
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + row * C);
    for (int i = lane; i < nq; i += 32) {
      uint2 o = make_uint2(0u, 0u);
      if (valid) {
        const float4 v = __ldg(src + i);
        o.x = pack_bf16x2(__fdiv_rn(v.x, d), __fdiv_rn(v.y, d));
        o.y = pack_bf16x2(__fdiv_rn(v.z, d), __fdiv_rn(v.w, d));
      }
      dst[i] = o;
    }
  } else {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row * C);
    for (int i = lane; i < nq; i += 32) {
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (valid) {
        const float4 v = __ldg(src + i);
        o = make_float4(__fdiv_rn(v.x, d), __fdiv_rn(v.y, d), __fdiv_rn(v.z, d), __fdiv_rn(v.w, d));
      }
      dst[i] = o;
    }
  }
}

cudaError_t launch_norm(const float* rows, const uint8_t* mask, long long nrows, int C, float eps,
                        bool out_bf16, void* out, cudaStream_t stream) {
  if (nrows == 0) return cudaSuccess;
  const int rows_per_block = 8;
  const long long blocks = (nrows + rows_per_block - 1) / rows_per_block;
  if (out_bf16)
    norm_rows_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(rows, mask, nrows, C, eps, out);
  else
    norm_rows_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(rows, mask, nrows, C, eps, out);
  return cudaGetLastError();
}

}  // namespace gkd
