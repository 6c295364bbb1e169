// Step a2: L2 normalisation of prompt rows: the head normalises each kernel row
// to unit L2 norm (GKD_GGUF model card, Model section, Architecture bullet; the
// convolution with prompts is a normalised one, GKDT reading notes, Method
// section). One warp per row: 128-bit loads, fp32 sum of squares, warp-shuffle
// reduction, IEEE sqrt and division, optional round-to-nearest-even bf16 output.
#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {

constexpr int kNormRegQ = 10;   // float4 per lane held in registers: rows of up to 1280 channels

template <bool OUT_BF16>
__device__ __forceinline__ void store_norm(void* out, long long row, int C, int i, const float4& v, float d,
                                           bool valid) {
  if (OUT_BF16) {
    uint2 o = make_uint2(0u, 0u);
    if (valid) {
      o.x = pack_bf16x2(__fdiv_rn(v.x, d), __fdiv_rn(v.y, d));
      o.y = pack_bf16x2(__fdiv_rn(v.z, d), __fdiv_rn(v.w, d));
    }
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + row * C)[i] = o;
  } else {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) o = make_float4(__fdiv_rn(v.x, d), __fdiv_rn(v.y, d), __fdiv_rn(v.z, d), __fdiv_rn(v.w, d));
    reinterpret_cast<float4*>(static_cast<float*>(out) + row * C)[i] = o;
  }
}

// One warp per row. Rows of up to 1280 channels are read once: every lane
// issues all of its 128-bit loads before the first use, keeps them in
// registers for the division pass, and sums its squares in channel order
// (lane, lane + 32, ...), as the streaming loop for longer rows does.
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
  const bool in_regs = nq <= 32 * kNormRegQ;
  float4 reg[kNormRegQ];
  float ss = 0.f;
  if (valid) {
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kNormRegQ; ++j) {
        const int i = lane + 32 * j;
        reg[j] = i < nq ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < kNormRegQ; ++j) {
        if (lane + 32 * j < nq) {
          ss = fmaf(reg[j].x, reg[j].x, ss);
          ss = fmaf(reg[j].y, reg[j].y, ss);
          ss = fmaf(reg[j].z, reg[j].z, ss);
          ss = fmaf(reg[j].w, reg[j].w, ss);
        }
      }
    } else {
      for (int i = lane; i < nq; i += 32) {
        const float4 v = __ldg(src + i);
        ss = fmaf(v.x, v.x, ss);
        ss = fmaf(v.y, v.y, ss);
        ss = fmaf(v.z, v.z, ss);
        ss = fmaf(v.w, v.w, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const float d = fmaxf(__fsqrt_rn(ss), eps);
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kNormRegQ; ++j) {
      const int i = lane + 32 * j;
      if (i < nq) store_norm<OUT_BF16>(out, row, C, i, reg[j], d, valid);
    }
  } else {
    for (int i = lane; i < nq; i += 32)
      store_norm<OUT_BF16>(out, row, C, i, valid ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f), d, valid);
  }
}

// Modality fusion moved before the contraction (the heatmap is linear in the
// kernel row, so the mean of a prompt row's modality heatmaps, GKD_GGUF model
// card, Model section, Architecture and Prompts bullets, is the heatmap of the
// mean of its normalised rows). One warp per output row (crop, k): each present
// modality's row is normalised as in norm_rows_kernel, the present ones are
// averaged in fp32 ((a + b) * 0.5, or the one row unchanged), and the result is
// rounded once (to bf16) on output. out_mask[b,k] = any modality present.
template <bool OUT_BF16>
__global__ void __launch_bounds__(256) norm_fuse_kernel(const float* __restrict__ rows,
                                                        const uint8_t* __restrict__ mask, long long nout, int M,
                                                        int K, int C, float eps, void* __restrict__ out,
                                                        uint8_t* __restrict__ out_mask) {
  const int lane = threadIdx.x & 31;
  const long long o = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (o >= nout) return;
  const long long b = o / K;
  const int k = static_cast<int>(o % K);
  const int nq = C >> 2;
  const float4* src0 = reinterpret_cast<const float4*>(rows + ((b * M) * K + k) * C);
  const float4* src1 = reinterpret_cast<const float4*>(rows + ((b * M + 1) * K + k) * C);
  const bool p0 = mask[(b * M) * K + k] != 0;
  const bool p1 = M == 2 && mask[(b * M + 1) * K + k] != 0;
  float s0 = 0.f, s1 = 0.f;
  for (int i = lane; i < nq; i += 32) {
    if (p0) {
      const float4 v = __ldg(src0 + i);
      s0 = fmaf(v.x, v.x, s0);
      s0 = fmaf(v.y, v.y, s0);
      s0 = fmaf(v.z, v.z, s0);
      s0 = fmaf(v.w, v.w, s0);
    }
    if (p1) {
      const float4 v = __ldg(src1 + i);
      s1 = fmaf(v.x, v.x, s1);
      s1 = fmaf(v.y, v.y, s1);
      s1 = fmaf(v.z, v.z, s1);
      s1 = fmaf(v.w, v.w, s1);
    }
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) {
    s0 += __shfl_xor_sync(0xffffffffu, s0, sh);
    s1 += __shfl_xor_sync(0xffffffffu, s1, sh);
  }
  const float d0 = fmaxf(__fsqrt_rn(s0), eps), d1 = fmaxf(__fsqrt_rn(s1), eps);
  if (lane == 0) out_mask[o] = (p0 || p1) ? 1 : 0;
  for (int i = lane; i < nq; i += 32) {
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p0 || p1) {
      float4 a = f, c = f;
      if (p0) {
        const float4 v = __ldg(src0 + i);
        a = make_float4(__fdiv_rn(v.x, d0), __fdiv_rn(v.y, d0), __fdiv_rn(v.z, d0), __fdiv_rn(v.w, d0));
      }
      if (p1) {
        const float4 v = __ldg(src1 + i);
        c = make_float4(__fdiv_rn(v.x, d1), __fdiv_rn(v.y, d1), __fdiv_rn(v.z, d1), __fdiv_rn(v.w, d1));
      }
      if (p0 && p1)
        f = make_float4(__fmul_rn(__fadd_rn(a.x, c.x), 0.5f), __fmul_rn(__fadd_rn(a.y, c.y), 0.5f),
                        __fmul_rn(__fadd_rn(a.z, c.z), 0.5f), __fmul_rn(__fadd_rn(a.w, c.w), 0.5f));
      else
        f = p0 ? a : c;
    }
    if (OUT_BF16) {
      reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + o * C)[i] =
          make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
    } else {
      reinterpret_cast<float4*>(static_cast<float*>(out) + o * C)[i] = f;
    }
  }
}

cudaError_t launch_norm_fuse(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C, float eps,
                             bool out_bf16, void* out, uint8_t* out_mask, cudaStream_t stream) {
  const long long nout = static_cast<long long>(Bk) * K;
  if (nout == 0) return cudaSuccess;
  const long long blocks = (nout + 7) / 8;
  if (out_bf16)
    norm_fuse_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(rows, mask, nout, M, K, C, eps, out,
                                                                              out_mask);
  else
    norm_fuse_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(rows, mask, nout, M, K, C, eps, out,
                                                                               out_mask);
  return cudaGetLastError();
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
