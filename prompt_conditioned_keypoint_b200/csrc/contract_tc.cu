// Contract-then-upsample variant of steps a3 + a4 (the 1x1 contraction and the
// 4x bilinear upsample are both linear, so their order can be swapped: GKD_GGUF
// model card, Model section, Architecture bullet lists them; the graded path
// keeps upsample-then-contract). Two kernels:
//
//   contract_kernel  G[b,m,k,i,j] = sum_c khat[b,m,k,c] * bf16(F[b,i,j,c]) on the
//                    h x w source grid: a tcgen05 GEMM per (crop, tile of 128
//                    source pixels), M = pixels, N = the crop's valid rows, K = C.
//                    Two groups of four warps take the 64-channel stages in
//                    turn and turn each TMA-loaded slab into the bf16 A
//                    operand in tensor memory (one pixel per lane: fp32
//                    features rounded to nearest even, bf16 features copied);
//                    TMA brings the kernel rows as the B operand; the fp32
//                    accumulator is written to G, one row of the crop at a time.
//   upsample_kernel  heat[b,m,k] = the 4x bilinear upsample (align_corners=False,
//                    half-pixel rule, borders clamped) of G[b,m,k] in fp32:
//                    x-lerps on the two source rows, then the y-lerp.
//
// 16x fewer multiply-adds than the graded path; the heatmap writes dominate, so
// the pair is bound by HBM. One CTA per unit (no persistence): the GEMM is small,
// so each CTA takes half an SM (104 KB of shared memory, 256 tensor-memory
// columns) and two CTAs overlap each other's load latency.
// Every wait is bounded; on a timeout the CTA records it and drains.
#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {
namespace cf {

constexpr int kStages = 2;                          // ring of 64-channel stages (two CTAs share an SM)
constexpr int kChunk = 64;
constexpr int kMaxN = 160;
constexpr int kTile = 128;                          // source pixels per unit (TMEM lanes)
constexpr int kFeatBytes = kTile * 256;             // fp32: two 128-byte planes per pixel (bf16 uses one)
constexpr int kBBytes = kMaxN * 128;                // kernel rows of a stage, 64 bf16 channels each
constexpr int kWarps = 10;                          // 0 TMA, 1 MMA, 2-9 convert + epilogue (two groups of four)
constexpr int kConvGroups = 2;                      // group g converts the stages s with s % 2 == g
static_assert(kConvGroups == kStages, "a converter group owns one ring slot");
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kTmemCols = 256;                 // accumulator (<= 160) + two 32-column A stages
constexpr uint32_t kColA = kMaxN;                   // accumulator at 0, A stages at 160 + 32 s
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * (kFeatBytes + kBBytes) + 256;

struct Ctl {
  uint64_t full[kStages];    // features + kernel rows landed
  uint64_t aready[kStages];  // A operand written (4 converter warps)
  uint64_t empty[kStages];   // MMA done with the stage
  uint64_t accfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Seg {
  int kmin[2], len[2], off1, n;
};

// Warp-cooperative (every lane gets the result): the valid-row segment of each
// modality. Lane l reads mask bytes 8l .. 8l+7 of the crop's [M][K] mask (M K <=
// 256), so the whole mask costs one memory latency.
__device__ __forceinline__ Seg segments(const ContractArgs& a, const uint8_t* mb, int lane) {
  Seg g{};
  const int total = a.M * a.K;
  uint32_t lb = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = 8 * lane + i;
    if (p < total && mb[p] != 0) lb |= 1u << i;
  }
  int off = 0;
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    g.kmin[m] = 0;
    g.len[m] = 0;
    if (m < a.M) {
      int first = a.K, last = -1;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int k = 8 * lane + i - m * a.K;
        if (((lb >> i) & 1u) && k >= 0 && k < a.K) {
          first = min(first, k);
          last = max(last, k);
        }
      }
      first = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<unsigned>(first)));
      last = __reduce_max_sync(0xffffffffu, last);
      if (last >= 0) {
        g.kmin[m] = first;
        g.len[m] = (last - first + 1 + 7) & ~7;
      }
    }
    if (m == 0) g.off1 = g.len[0];
    off += g.len[m];
  }
  g.n = (off + 15) & ~15;
  return g;
}

__device__ __forceinline__ uint32_t make_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ uint64_t make_bdesc(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__global__ void __launch_bounds__(kThreads, 2) contract_kernel(const __grid_constant__ ContractArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bring = smem + kStages * kFeatBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(bring + kStages * kBBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hw = a.h * a.w;
  const int ntiles = (hw + kTile - 1) / kTile;
  const int b = blockIdx.x / ntiles, tile = blockIdx.x % ntiles;
  const int px0 = tile * kTile;
  const uint8_t* mb = a.mask + static_cast<long long>(b) * a.mask_batch_stride;
  const Seg sg = segments(a, mb, threadIdx.x & 31);
  if (sg.n == 0) return;                              // uniform: no valid row in this crop
  const int nst = (a.C + kChunk - 1) / kChunk;
  const uint64_t lim = a.wait_limit_ns;
  volatile int* abortp = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->aready[s], 4);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA: feature slab + kernel rows
    uint32_t it = 0;
    bool ok = true;
    const int bk = a.kern_shared ? 0 : b;
    const uint32_t fbytes = (a.feat_bf16 ? 128u : 256u) * kTile;
    const uint32_t bytes = fbytes + 2u * (sg.len[0] + sg.len[1]) * 64u;
    for (; it < static_cast<uint32_t>(nst) && ok; ++it) {
      const uint32_t s = it % kStages, ph = (it / kStages) & 1;
      const bool okw = it < kStages || mbar_wait_bounded(&ctl->empty[s], ph ^ 1, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) {
          ctl->abort_flag = 1;
          atomicOr(a.err, kErrTimeout);
        }
        ok = false;
        break;
      }
      if (lane == 0) {
        uint64_t* fb = &ctl->full[s];
        mbar_arrive_expect_tx(fb, bytes);
        const int c0 = static_cast<int>(it) * kChunk;
        uint8_t* fp = smem + s * kFeatBytes;
        const int row = b * hw + px0;
        if (a.feat_bf16) {
          tma_load_2d(fp, &a.tmap_feat, fb, c0, row);
        } else {
          tma_load_2d(fp, &a.tmap_feat, fb, c0, row);
          tma_load_2d(fp + kTile * 128, &a.tmap_feat, fb, c0 + 32, row);
        }
        uint8_t* bp = bring + s * kBBytes;
        if (sg.len[0]) tma_load_4d(bp, &a.tmap_kern[(sg.len[0] >> 3) - 1], fb, c0, sg.kmin[0], 0, bk);
        if (sg.len[1])
          tma_load_4d(bp + sg.off1 * 128, &a.tmap_kern[(sg.len[1] >> 3) - 1], fb, c0, sg.kmin[1], 1, bk);
      }
      __syncwarp();
    }
    if (lane == 0)
      for (uint32_t k = 0; k < kStages && k < it; ++k) {
        const uint32_t last = it - 1 - k;
        if (!mbar_wait_drain(&ctl->full[last % kStages], (last / kStages) & 1, lim)) atomicOr(a.err, kErrTimeout);
      }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA (one thread)
    if (lane == 0) {
      const uint32_t idesc = make_idesc(sg.n);
      const uint64_t bdesc0 = make_bdesc(smem_u32(bring));
      uint32_t it = 0;
      bool ok = true;
      for (; it < static_cast<uint32_t>(nst); ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1;
        if (!mbar_wait_bounded(&ctl->aready[s], ph, lim, abortp)) {
          ctl->abort_flag = 1;
          atomicOr(a.err, kErrTimeout);
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts_f16(tmem, tmem + kColA + s * 32 + kk * 8,
                      bdesc0 + static_cast<uint64_t>((s * kBBytes + kk * 32) >> 4), idesc,
                      (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&ctl->empty[s]);
      }
      if (ok) umma_commit(&ctl->accfull);
      if (it > 0) {
        umma_commit(&ctl->drain);
        if (!mbar_wait_drain(&ctl->drain, 0, lim)) atomicOr(a.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ convert, then epilogue
    const int q = warp & 3;                           // lane quadrant
    const int grp = (warp - 2) >> 2;                  // converter group: stages grp, grp + 2, ...
    const int r = 32 * q + lane;                      // tile pixel of this thread
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    bool ok = true;
    // the two groups alternate stages, so one group's TMEM-store wait overlaps
    // the other group's conversion
    for (uint32_t it = grp; it < static_cast<uint32_t>(nst); it += kConvGroups) {
      const uint32_t s = it % kStages, ph = (it / kStages) & 1;
      const bool okw = mbar_wait_bounded(&ctl->full[s], ph, lim, abortp);
      if (!__all_sync(0xffffffffu, okw)) {
        if (lane == 0) {
          ctl->abort_flag = 1;
          atomicOr(a.err, kErrTimeout);
        }
        ok = false;
        break;
      }
      const uint32_t fp = smem_u32(smem + s * kFeatBytes) + r * 128u;
      uint32_t v[32];
      if (a.feat_bf16) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t x, y, z, w4;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(x), "=r"(y), "=r"(z), "=r"(w4)
                       : "r"(fp + ((static_cast<uint32_t>(j) ^ (r & 7u)) << 4)));
          v[4 * j] = x;
          v[4 * j + 1] = y;
          v[4 * j + 2] = z;
          v[4 * j + 3] = w4;
        }
      } else {
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float x, y, z, w4;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(x), "=f"(y), "=f"(z), "=f"(w4)
                         : "r"(fp + pl * kTile * 128u + ((static_cast<uint32_t>(j) ^ (r & 7u)) << 4)));
            v[16 * pl + 2 * j] = pack_bf16x2(x, y);
            v[16 * pl + 2 * j + 1] = pack_bf16x2(z, w4);
          }
        }
      }
      tmem_st_32x32b_x32(tmem + lane_off + kColA + s * 32, v);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->aready[s]);
    }
    // epilogue: accumulator column n -> G row of (m, k); one pixel per lane
    const bool okw = ok && mbar_wait_bounded(&ctl->accfull, 0, lim, abortp);
    if (__all_sync(0xffffffffu, okw)) {
      tc_fence_after();
      const bool pix_ok = px0 + r < hw;
      // valid accumulator columns as bits (bit c of word g: column 32 g + c), one
      // mask byte per lane and word, so the loop below reads no mask
      uint32_t colw[5];
#pragma unroll
      for (int g = 0; g < 5; ++g) {
        const int n = 32 * g + lane;
        const int m = n < sg.off1 ? 0 : 1;
        const int k = (m ? sg.kmin[1] : sg.kmin[0]) + n - (m ? sg.off1 : 0);
        const bool v = n < sg.len[0] + sg.len[1] && k < a.K && mb[m * a.K + k] != 0;
        colw[g] = __ballot_sync(0xffffffffu, v);
      }
      float* gcrop = a.G + static_cast<long long>(b) * a.M * a.K * hw + px0 + r;
      for (int n0 = 16 * grp; n0 < sg.n; n0 += 16 * kConvGroups) {   // the groups take alternate 16-column chunks
        uint32_t vv[16];
        tmem_ld_32x32b_x16(tmem + lane_off + n0, vv);
        tmem_wait_ld();
        const int g = n0 >> 5;   // select without indexing (keeps colw in registers)
        const uint32_t word = g == 0 ? colw[0] : g == 1 ? colw[1] : g == 2 ? colw[2] : g == 3 ? colw[3] : colw[4];
        const uint32_t bits = (word >> (n0 & 31)) & 0xFFFFu;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int n = n0 + c;
          const int m = n < sg.off1 ? 0 : 1;
          const int k = (m ? sg.kmin[1] : sg.kmin[0]) + n - (m ? sg.off1 : 0);
          if (((bits >> c) & 1u) && pix_ok)
            gcrop[(static_cast<long long>(m) * a.K + k) * hw] = __uint_as_float(vv[c]);
        }
      }
    } else if (lane == 0) {
      ctl->abort_flag = 1;
      atomicOr(a.err, kErrTimeout);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// heat[b,m,k] = Up(G[b,m,k]) for valid rows; one CTA per (crop, row): the row's
// source-grid map is staged in shared memory once (read in place from global
// memory when it does not fit, STAGED = false). A thread's work item is a band
// of four output rows (Y = 4s+2 .. 4s+5, which all read source rows s and s+1,
// clamped at the borders) by four consecutive output columns: it x-lerps the
// four columns on the two source rows once and y-lerps them into the band's
// rows, one float4 (streaming) per row. The arithmetic per pixel is that of
// the plain rule: x-lerps on the two source rows, then the y-lerp.
template <bool STAGED>
__global__ void __launch_bounds__(256) upsample_kernel(const float* __restrict__ G, const uint8_t* __restrict__ mask,
                                                       long long mask_bs, int M, int K, int h, int w,
                                                       float* __restrict__ heat) {
  extern __shared__ float gsm[];                         // [h][w] when staged
  const int row = blockIdx.x, b = blockIdx.y;          // row = m * K + k
  if (!mask[static_cast<long long>(b) * mask_bs + row]) return;
  const int H = 4 * h, W = 4 * w;
  const float* g = G + (static_cast<long long>(b) * M * K + row) * h * w;
  const float* gs = g;
  if (STAGED) {
    for (int e = threadIdx.x; e < h * w; e += blockDim.x) gsm[e] = __ldg(g + e);
    __syncthreads();
    gs = gsm;
  }
  float* out = heat + (static_cast<long long>(b) * M * K + row) * static_cast<long long>(H) * W;
  const int nitems = (h + 1) * w;                      // bands x float4 columns
  for (int it = threadIdx.x; it < nitems; it += blockDim.x) {
    const int band = it / w, u = it - band * w;
    const int Yb = 4 * band - 2;                        // the band's first output row (may be < 0)
    // source rows of the band, from its first row inside the map
    const int Yf = max(Yb, 0);
    const float sy0 = fmaxf((static_cast<float>(Yf) + 0.5f) * 0.25f - 0.5f, 0.f);
    const int i0 = static_cast<int>(sy0), i1 = min(i0 + 1, h - 1);
    const float* r0 = gs + i0 * w;
    const float* r1 = gs + i1 * w;
    float t0[4], t1[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int X = 4 * u + e;
      const float sx = fmaxf((static_cast<float>(X) + 0.5f) * 0.25f - 0.5f, 0.f);
      const int j0 = static_cast<int>(sx), j1 = min(j0 + 1, w - 1);
      const float lx = sx - static_cast<float>(j0);
      t0[e] = fmaf(lx, r0[j1] - r0[j0], r0[j0]);
      t1[e] = fmaf(lx, r1[j1] - r1[j0], r1[j0]);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int Y = Yb + t;
      if (Y < 0 || Y >= H) continue;
      const float sy = fmaxf((static_cast<float>(Y) + 0.5f) * 0.25f - 0.5f, 0.f);
      const float ly = sy - static_cast<float>(i0);
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = fmaf(ly, t1[e] - t0[e], t0[e]);
      __stcs(reinterpret_cast<float4*>(out + static_cast<long long>(Y) * W) + u, make_float4(v[0], v[1], v[2], v[3]));
    }
  }
}

}  // namespace cf

static bool encode_sw128(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                         const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_contract_first(ContractArgs& a, const void* feat, const void* kern, long long kern_batch_stride,
                                  float* heat, cudaStream_t stream, const char** why) {
  if (a.B == 0) return cudaSuccess;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) {
    *why = "cuTensorMapEncodeTiled is unavailable";
    return cudaErrorNotSupported;
  }
  const cuuint64_t C = a.C, npx = static_cast<cuuint64_t>(a.B) * a.h * a.w;
  {
    const cuuint64_t elt = a.feat_bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {C, npx};
    const cuuint64_t strides[1] = {C * elt};
    const cuuint32_t box[2] = {a.feat_bf16 ? 64u : 32u, static_cast<cuuint32_t>(cf::kTile)};
    if (!encode_sw128(enc, &a.tmap_feat, a.feat_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      2, feat, dims, strides, box)) {
      *why = "tensor map encoding failed for the feature map";
      return cudaErrorInvalidValue;
    }
  }
  {
    const cuuint64_t Bk = a.kern_shared ? 1 : static_cast<cuuint64_t>(a.B);
    const cuuint64_t K = a.K, M = a.M;
    const cuuint64_t bstride = a.kern_shared ? M * K * C * 2 : static_cast<cuuint64_t>(kern_batch_stride) * 2;
    const cuuint64_t dims[4] = {C, K, M, Bk};
    const cuuint64_t strides[3] = {C * 2, K * C * 2, bstride};
    for (int i = 0; i < kKernMaps; ++i) {
      const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(8 * (i + 1)), 1, 1};
      if (!encode_sw128(enc, &a.tmap_kern[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kern, dims, strides, box)) {
        *why = "tensor map encoding failed for the kernel rows";
        return cudaErrorInvalidValue;
      }
    }
  }
  cudaError_t e = cudaFuncSetAttribute(cf::contract_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(cf::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int ntiles = (a.h * a.w + cf::kTile - 1) / cf::kTile;
  const long long grid = static_cast<long long>(a.B) * ntiles;
  cf::contract_kernel<<<static_cast<unsigned>(grid), cf::kThreads, cf::kSmemBytes, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(a.M * a.K, a.B);
  const size_t gsmem = sizeof(float) * static_cast<size_t>(a.h) * a.w;
  if (gsmem <= 96 * 1024) {
    if (gsmem > 48 * 1024) {
      e = cudaFuncSetAttribute(cf::upsample_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(gsmem));
      if (e != cudaSuccess) return e;
    }
    cf::upsample_kernel<true><<<g2, 256, gsmem, stream>>>(a.G, a.mask, a.mask_batch_stride, a.M, a.K, a.h, a.w,
                                                          heat);
  } else {
    cf::upsample_kernel<false><<<g2, 256, 0, stream>>>(a.G, a.mask, a.mask_batch_stride, a.M, a.K, a.h, a.w, heat);
  }
  return cudaGetLastError();
}

}  // namespace gkd
