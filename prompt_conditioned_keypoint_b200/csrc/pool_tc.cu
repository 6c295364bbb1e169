// Step a1 on the tensor cores: Gaussian prototype pooling (visual prompts are
// one-shot keypoints pooled with a Gaussian of sigma 14 px: GKD_GGUF model card,
// Model section, Prompts bullet; prototypes from Gaussian weights placed on the
// support image at the keypoints: GKDT summary page, pipeline paragraph).
//
//   proto[b,k,:] = sum_p w[k,p] F[b,p,:] / sum_p w[k,p],
//   w[k,p] = exp(-((X_j - x)^2 + (Y_i - y)^2 - d2min) / (2 sigma^2)), p = (i, j),
//
// is one GEMM per crop: M = the keypoints (K <= 128, one M=128 tile), N = the
// channels, and the reduction runs over the crop's h*w pixels. It runs as
// tcgen05.mma kind::tf32 with fp32 accumulation in tensor memory. d2min (the
// squared distance to the nearest patch centre) is a common factor of every
// weight of a keypoint and cancels in the ratio; it keeps the largest weight at
// exactly 1 so the normaliser never underflows.
//
// fp32 accuracy from TF32 operands: every operand x is split as x = hi + lo
// with hi = x rounded to TF32 (11 significant bits) and lo = x - hi (exact in
// fp32); w F is taken as w_hi F_hi + w_hi F_lo + w_lo F_hi. The dropped term
// w_lo F_lo and the rounding of lo to TF32 are each below 2^-21 of |w F|.
//
// One CTA per (crop, block of N <= 256 channels), 14 warps:
//   warp 0      TMA: per stage of 32 pixels, the [32 px][N ch] fp32 feature tile
//               (boxes of 32 pixels x 32 channels; pixels past h*w and channels
//               past C read as zeros) into a 3-deep raw ring;
//   warp 1      MMA: per stage, 4 K-steps x 3 products, into an N-column fp32
//               accumulator; one commit frees the stage;
//   warps 2-5   weights (one thread per keypoint = tensor-memory lane): the
//               stage's 32 weights of its keypoint, split hi/lo, stored as the
//               A operand (tcgen05.st.32x32b.x32, hi and lo 32 columns each);
//               they also sum the keypoint's weights in pixel order and, at the
//               end, scale and store the prototypes;
//   warps 6-13  converters (one thread per channel): the stage's raw tile split
//               hi/lo and transposed into two K-major, 128B-swizzled B tiles
//               (2-deep, as are the A stages in tensor memory).
// Every wait is bounded; a timeout sets the device error word and every role
// drains what it has in flight.
#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {
namespace ptc {

constexpr int kMaxN = 256;                         // channels per CTA at most (accumulator columns)
constexpr int kKs = 32;                            // pixels per stage: one 128-byte row of tf32 per channel
constexpr int kRawStages = 3;                      // raw feature tiles (TMA -> converters)
constexpr int kStages = 2;                         // B tiles in shared memory and A stages in tensor memory
constexpr int kBoxBytes = kKs * 32 * 4;            // one TMA box: 32 pixels x 32 channels
constexpr int kRawBytes = kMaxN / 32 * kBoxBytes;  // 32 KB: [box][pixel][32 channels]
constexpr int kOpBytes = kMaxN * kKs * 4;          // 32 KB: one K-major operand tile [channel][32 px], swizzled
constexpr int kBStageBytes = 2 * kOpBytes;         // B_hi then B_lo
constexpr int kBRingOffset = kRawStages * kRawBytes;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpW0 = 2, kNumWWarps = 4, kWarpCv0 = 6, kNumCvWarps = 8;
constexpr int kNumWarps = kWarpCv0 + kNumCvWarps, kThreads = kNumWarps * 32;
constexpr uint32_t kTmemCols = 512;                // accumulator at 0..N-1, A stages at 256 + 64 s
constexpr uint32_t kColA = 256;
static_assert(kNumCvWarps * 32 == kMaxN, "one converter thread per channel");
static_assert(kWarpW0 + kNumWWarps == kWarpCv0 && kNumWWarps * 32 == 128, "one weight thread per keypoint lane");

struct Ctl {
  uint64_t rfull[kRawStages];   // raw tile landed (TMA bytes)
  uint64_t rempty[kRawStages];  // raw tile read by every converter warp
  uint64_t bready[kStages];   // B tiles written (converter warps)
  uint64_t aready[kStages];   // A stage written (weight warps)
  uint64_t sempty[kStages];   // MMA done with the stage's A and B
  uint64_t accfull;           // every MMA done
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kBRingOffset) + static_cast<size_t>(kStages) * kBStageBytes + 256;
static_assert(sizeof(Ctl) <= 256, "control block");

__device__ __forceinline__ uint32_t tf32_hi(float x) {   // x rounded to TF32, as an fp32 bit pattern
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {   // 2^x (hardware approximation, about 2^-22 relative)
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint64_t make_bdesc(uint32_t smem_addr) {
  // K-major, 128B swizzle: LBO = 1 (16 B), SBO = 1024 B (8 rows x 128 B), version 1, layout 2.
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ uint32_t make_idesc_tf32(int n) {
  // kind::tf32: D fp32 (bit 4), A and B tf32 (bits 7-9 and 10-12 = 2), both
  // K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28 (M = 128).
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void set_abort(Ctl* ctl, unsigned* err) {
  ctl->abort_flag = 1;
  atomicOr(err, kErrTimeout);
}

__device__ __forceinline__ float nearest_d2(float x, float stride, int n) {
  // squared distance from x to the nearest of the centres stride (j + 0.5), j = 0..n-1
  const float t = x / stride - 0.5f;
  const int j0 = min(max(static_cast<int>(floorf(t)), 0), n - 1);
  const int j1 = min(j0 + 1, n - 1);
  const float d0 = stride * (static_cast<float>(j0) + 0.5f) - x;
  const float d1 = stride * (static_cast<float>(j1) + 0.5f) - x;
  return fminf(d0 * d0, d1 * d1);
}

__global__ void __launch_bounds__(kThreads, 1) pool_tc_kernel(const __grid_constant__ PoolTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + kBRingOffset + kStages * kBStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, c0 = blockIdx.x * a.N;
  const int P = a.h * a.w;
  const int nstages = (P + kKs - 1) / kKs;
  const uint64_t lim = a.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&ctl->rfull[s], 1);
      mbar_init(&ctl->rempty[s], kNumCvWarps);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->bready[s], kNumCvWarps);
      mbar_init(&ctl->aready[s], kNumWWarps);
      mbar_init(&ctl->sempty[s], 1);
    }
    mbar_init(&ctl->accfull, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) tma_prefetch_desc(&a.tmap);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  volatile int* abortp = &ctl->abort_flag;
  const bool run = tmem == 0;   // the column offsets below assume the allocation starts at column 0
  if (threadIdx.x == 0 && !run) atomicOr(a.err, kErrBounds);

  if (warp == kWarpTma) {
    // ------------------------------------------------------------------ TMA
    const int nbox = a.N / 32;
    int s = 0;
    bool ok = run;
    for (; ok && s < nstages; ++s) {
      const int rs = s % kRawStages;
      const bool okw = s < kRawStages ||
                       mbar_wait_bounded(&ctl->rempty[rs], ((s / kRawStages) & 1) ^ 1, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) set_abort(ctl, a.err);
        ok = false;
        break;
      }
      if (lane == 0) {
        uint8_t* raw = smem + rs * kRawBytes;
        mbar_arrive_expect_tx(&ctl->rfull[rs], static_cast<uint32_t>(nbox * kBoxBytes));
        for (int bx = 0; bx < nbox; ++bx)
          tma_load_3d(raw + bx * kBoxBytes, &a.tmap, &ctl->rfull[rs], c0 + 32 * bx, s * kKs, b);
      }
      __syncwarp();
    }
    // drain: the last loads issued have landed before the CTA exits
    if (lane == 0) {
      for (int k = 0; k < kRawStages && k < s; ++k) {
        const int last = s - 1 - k;
        if (!mbar_wait_drain(&ctl->rfull[last % kRawStages], (last / kRawStages) & 1, lim))
          atomicOr(a.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA
    const uint32_t idesc = make_idesc_tf32(a.N);
    int s = 0;
    bool ok = run;
    for (; ok && s < nstages; ++s) {
      const int slot = s & 1;
      const uint32_t par = (s >> 1) & 1;
      const bool okw = mbar_wait_bounded(&ctl->bready[slot], par, lim, abortp) &&
                       mbar_wait_bounded(&ctl->aready[slot], par, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) set_abort(ctl, a.err);
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t bhi = smem_u32(smem + kBRingOffset + slot * kBStageBytes);
        const uint64_t dhi = make_bdesc(bhi), dlo = make_bdesc(bhi + kOpBytes);
        const uint32_t ahi = tmem + kColA + static_cast<uint32_t>(slot) * 64, alo = ahi + 32;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk * 32) >> 4);
          umma_tf32(tmem, ahi + 8 * kk, dhi + off, idesc, (s | kk) ? 1u : 0u);
          umma_tf32(tmem, ahi + 8 * kk, dlo + off, idesc, 1u);
          umma_tf32(tmem, alo + 8 * kk, dhi + off, idesc, 1u);
        }
        umma_commit(&ctl->sempty[slot]);
      }
      __syncwarp();
    }
    // the final commit: every MMA issued has completed (also on the abort path,
    // so that teardown never frees tensor memory under a running MMA)
    if (lane == 0) umma_commit(&ctl->accfull);
    __syncwarp();
  } else if (warp < kWarpCv0) {
    // ------------------------------------------------------------------ weights, then the prototypes
    const int q = warp & 3;                        // lane quadrant this warp may access
    const int k = 32 * q + lane;                   // keypoint = tensor-memory lane
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const bool valid = k < a.K && a.kmask[static_cast<long long>(b) * a.K + k] != 0;
    const float x = valid ? a.kpts[(static_cast<long long>(b) * a.K + k) * 2] : 0.f;
    const float y = valid ? a.kpts[(static_cast<long long>(b) * a.K + k) * 2 + 1] : 0.f;
    const float d2min = nearest_d2(x, a.stride, a.w) + nearest_d2(y, a.stride, a.h);
    // w = 2^(-(dx^2 + dy^2 - d2min) k2), k2 = log2(e) / (2 sigma^2); walking the
    // pixels in order, dx comes from a running column centre and the row's
    // (dy^2 - d2min) k2 is formed once per row (rows change at the same pixel
    // for every thread: a uniform branch)
    const float k2 = 1.4426950408889634f / (2.0f * a.sigma * a.sigma);
    const float wf = static_cast<float>(a.w);
    auto row_term = [&](float ci) {
      const float dy = fmaf(a.stride, ci, -y);
      return (dy * dy - d2min) * k2;
    };
    float cj = 0.5f, ci = 0.5f;                    // column and row of the next pixel, + 0.5
    float dyt = row_term(ci);
    float wsum = 0.f;
    int s = 0;
    bool ok = run;
    for (; ok && s < nstages; ++s) {
      const int slot = s & 1;
      const bool okw = s < kStages || mbar_wait_bounded(&ctl->sempty[slot], ((s >> 1) & 1) ^ 1, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) set_abort(ctl, a.err);
        ok = false;
        break;
      }
      const int rem = P - s * kKs;                 // pixels of the crop left from this stage on
      const bool full = rem >= kKs;
      uint32_t vh[32], vl[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float dx = fmaf(a.stride, cj, -x);
        float wv = ex2_approx(-fmaf(dx * k2, dx, dyt));
        if (!valid || (!full && t >= rem)) wv = 0.f;
        wsum += wv;
        const uint32_t hi = tf32_hi(wv);
        vh[t] = hi;
        vl[t] = __float_as_uint(__fsub_rn(wv, __uint_as_float(hi)));
        cj += 1.0f;
        if (cj > wf) {
          cj = 0.5f;
          ci += 1.0f;
          dyt = row_term(ci);
        }
      }
      tc_fence_after();
      const uint32_t acol = tmem + lane_off + kColA + static_cast<uint32_t>(slot) * 64;
      tmem_st_32x32b_x32(acol, vh);
      tmem_st_32x32b_x32(acol + 32, vl);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->aready[slot]);
    }
    // prototypes: wait for every MMA, scale by 1 / sum of weights, store
    const bool okw = ok && mbar_wait_bounded(&ctl->accfull, 0, lim, abortp);
    if (!__all_sync(0xffffffffu, okw)) {
      if (lane == 0 && ok) set_abort(ctl, a.err);
      // the MMA warp's final commit still lands before teardown
      if (lane == 0) mbar_wait_drain(&ctl->accfull, 0, lim);
      __syncwarp();
    } else {
      tc_fence_after();
      const float sc = valid ? 1.0f / wsum : 0.f;
      float* row = a.proto + static_cast<long long>(b) * a.proto_bs + static_cast<long long>(k) * a.C + c0;
      for (int cc = 0; cc < a.N / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_off + static_cast<uint32_t>(32 * cc), v);
        tmem_wait_ld();
        if (k < a.K) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int c = c0 + 32 * cc + 4 * t;
            if (c < a.C) {
              const float4 o = valid ? make_float4(__uint_as_float(v[4 * t]) * sc, __uint_as_float(v[4 * t + 1]) * sc,
                                                   __uint_as_float(v[4 * t + 2]) * sc,
                                                   __uint_as_float(v[4 * t + 3]) * sc)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
              *reinterpret_cast<float4*>(row + 32 * cc + 4 * t) = o;
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ converters
    const int n = (warp - kWarpCv0) * 32 + lane;   // channel within the block = B-operand row
    const bool active = n < a.N;
    const uint32_t row_off = static_cast<uint32_t>((n >> 3) * 1024 + (n & 7) * 128);
    int s = 0;
    bool ok = run;
    for (; ok && s < nstages; ++s) {
      const int slot = s & 1, rs = s % kRawStages;
      const uint32_t par = (s >> 1) & 1;
      bool okw = mbar_wait_bounded(&ctl->rfull[rs], (s / kRawStages) & 1, lim, abortp);
      if (okw && s >= kStages) okw = mbar_wait_bounded(&ctl->sempty[slot], par ^ 1, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) set_abort(ctl, a.err);
        ok = false;
        break;
      }
      if (active) {
        const float* raw = reinterpret_cast<const float*>(smem + rs * kRawBytes + (n >> 5) * kBoxBytes) + (n & 31);
        const uint32_t bhi = smem_u32(smem + kBRingOffset + slot * kBStageBytes) + row_off;
#pragma unroll
        for (int c = 0; c < 8; ++c) {              // 16-byte chunk c = pixels 4c .. 4c+3
          float f[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) f[t] = raw[(4 * c + t) * 32];
          uint32_t h[4], l[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            h[t] = tf32_hi(f[t]);
            l[t] = __float_as_uint(__fsub_rn(f[t], __uint_as_float(h[t])));
          }
          const uint32_t addr = bhi + ((static_cast<uint32_t>(c) ^ static_cast<uint32_t>(n & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[0]), "r"(h[1]), "r"(h[2]),
                       "r"(h[3]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr + kOpBytes), "r"(l[0]), "r"(l[1]),
                       "r"(l[2]), "r"(l[3]) : "memory");
        }
      }
      fence_proxy_async_smem();                    // the tiles are read by the tensor cores (async proxy)
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->rempty[rs]);
        mbar_arrive(&ctl->bready[slot]);
      }
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace ptc

cudaError_t launch_pool_tc(const float* support, int B, int h, int w, int C, const float* kpts,
                           const uint8_t* kmask, int K, float sigma, float stride, float* proto,
                           long long proto_batch_stride, unsigned* err, unsigned long long wait_limit_ns,
                           int num_sms, cudaStream_t stream, const char** why) {
  if (B == 0) return cudaSuccess;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) {
    *why = "cuTensorMapEncodeTiled is unavailable";
    return cudaErrorNotSupported;
  }
  PoolTcArgs a{};
  const cuuint64_t P = static_cast<cuuint64_t>(h) * w;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), P, static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(C) * 4, P * C * 4};
  const cuuint32_t box[3] = {32, ptc::kKs, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(&a.tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(support), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *why = "tensor map encoding failed for the support features";
    return cudaErrorInvalidValue;
  }
  // the widest channel block (<= 256, a multiple of 32); halved while the CTAs would fill at most half the SMs
  int N = ptc::kMaxN;
  while (N > 32 && 2LL * B * ((C + N - 1) / N) <= num_sms) N /= 2;
  a.h = h;
  a.w = w;
  a.C = C;
  a.K = K;
  a.N = N;
  a.sigma = sigma;
  a.stride = stride;
  a.kpts = kpts;
  a.kmask = kmask;
  a.proto = proto;
  a.proto_bs = proto_batch_stride;
  a.err = err;
  a.wait_limit_ns = wait_limit_ns;
  cudaError_t e = cudaFuncSetAttribute(ptc::pool_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(ptc::kSmemBytes));
  if (e != cudaSuccess) return e;
  dim3 grid((C + N - 1) / N, B);
  ptc::pool_tc_kernel<<<grid, ptc::kThreads, ptc::kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gkd
