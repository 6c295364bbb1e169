// Steps a3 + a4 in fp32 (fp32 operands, fp32 accumulation on the FMA pipe):
// bilinear 4x upsample (align_corners=False) fused into the 1x1 dynamic-kernel
// contraction (the head upsamples the features 4x bilinearly and applies the
// prompts as 1x1 convolution kernels, GKD_GGUF model card, Model section,
// Architecture bullet). Used when the kernel rows are fp32;
// the tensor cores' fp32-input mode (tf32) would not meet a 1e-5 relative bound.
//
// One CTA per (crop, 4x32-pixel tile, group of up to ROWS valid rows), 512
// threads: 4 channel quarters x 128 pixels. The channels go in rounds of four
// 32-channel chunks, one per quarter. Per round the CTA copies, with cp.async
// into a double buffer, each quarter's chunk of the tile's source patch (the 3
// source rows x 10 source columns every pixel of the tile reads) and of its
// rows; the copies of round r + 1 are in flight while round r computes (a
// deeper ring measured no faster on one crop and slower on large batches). A
// thread owns one pixel: it forms the pixel's upsampled slice of its quarter's
// chunk from the patch (4 taps, dyadic weights) and contracts it against the
// chunk's rows. The four partial sums of a pixel are added in quarter order
// through shared memory at the end (a fixed order: the result does not depend
// on scheduling). ROWS is 32, or 16 when the batch has too few tiles to fill
// the SMs twice (a single crop: twice the CTAs, each upsampling again); a
// crop's rows are split evenly over the groups it needs.
//
// Decode mode (`keys` non-null): a group holds ROWS/2 prompt rows with both
// modality slots side by side, so each thread fuses its pixel's two heatmap
// values in fp32 and the CTA merges one peak key per row into `keys` with
// atomicMax (decode_key.cuh); no heatmap is written.
#include "decode_key.cuh"
#include "gkd_internal.h"

namespace gkd {

constexpr int kF32Pix = 128;                       // pixels per CTA (4 x 32 tile)
constexpr int kF32Quarters = 4;                    // channel quarters per CTA
constexpr int kF32Threads = kF32Pix * kF32Quarters;
constexpr int kF32Chunk = 32;                      // channels per quarter and round
constexpr int kPatchRows = 3, kPatchCols = 10, kPatchLines = kPatchRows * kPatchCols;
constexpr int kLinePitch = kF32Chunk + 4;          // floats per patch line: 8 distinct lines of a warp hit 8 bank groups
constexpr int kPatchFloats = kPatchLines * kLinePitch;

template <int ROWS>
struct F32Buf {                                    // one round: every quarter's patch and row chunk
  float patch[kF32Quarters][kPatchFloats];
  float4 ks[kF32Quarters][ROWS][kF32Chunk / 4];
};

template <int ROWS>
constexpr size_t f32_smem_bytes() {   // the double buffer, or the partial sums that reuse it if larger
  return 2 * sizeof(F32Buf<ROWS>) > sizeof(float) * (kF32Quarters - 1) * ROWS * kF32Pix
             ? 2 * sizeof(F32Buf<ROWS>)
             : sizeof(float) * (kF32Quarters - 1) * ROWS * kF32Pix;
}

__device__ __forceinline__ void taps_f32(int d, int n, int& i0, int& i1, float& lam) {
  const float s = fmaxf((static_cast<float>(d) + 0.5f) * 0.25f - 0.5f, 0.0f);
  i0 = min(static_cast<int>(s), n - 1);
  i1 = min(i0 + 1, n - 1);
  lam = s - static_cast<float>(static_cast<int>(s));
}

// 16-byte asynchronous copy global -> shared; `full` false: 16 zero bytes
// (nothing is read; `src` is still a valid address).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool full) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(full ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int ROWS>
__global__ void __launch_bounds__(kF32Threads) heatmap_f32_kernel(
    const float* __restrict__ feat, int h, int w, int C, const float* __restrict__ kern, long long kern_bs,
    const uint8_t* __restrict__ mask, long long mask_bs, int M, int K, float* __restrict__ heat,
    unsigned long long* __restrict__ keys) {
  __shared__ int rows[256];
  __shared__ int krow[128];
  __shared__ int s_nrows;
  extern __shared__ float4 f32_smem[];
  F32Buf<ROWS>* buf = reinterpret_cast<F32Buf<ROWS>*>(f32_smem);
  // partial sums of quarters 1..3, over the buffers once the last round is done
  float (*red)[ROWS][kF32Pix] = reinterpret_cast<float (*)[ROWS][kF32Pix]>(f32_smem);

  const int b = blockIdx.z, rg = blockIdx.y;
  const int H = 4 * h, W = 4 * w;
  const int ncb = (W + 31) / 32;
  const int band = blockIdx.x / ncb, cb = blockIdx.x % ncb;
  const uint8_t* mb = mask + static_cast<long long>(b) * mask_bs;
  const bool decode = keys != nullptr;
  if (threadIdx.x < 32) {
    // warp 0 lists the crop's valid rows in order: one ballot per 32 mask bytes,
    // each lane placing its row at the count of valid rows before it (M K <= 256)
    const int lane = threadIdx.x;
    const uint32_t below = (1u << lane) - 1u;
    int n = 0;
    if (!decode) {
      const int total = M * K;
      bool v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 32 * i + lane < total && mb[32 * i + lane] != 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t bal = __ballot_sync(0xffffffffu, v[i]);
        if (v[i]) rows[n + __popc(bal & below)] = 32 * i + lane;
        n += __popc(bal);
      }
    } else {
      // slots 2i, 2i+1: modality 0 and 1 of the i-th prompt row with any modality present (-1: absent)
      for (int k0 = 0; k0 < K; k0 += 32) {
        const int k = k0 + lane;
        const bool p0 = k < K && mb[k] != 0, p1 = k < K && M == 2 && mb[K + k] != 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, p0 || p1);
        if (p0 || p1) {
          const int i = n + __popc(bal & below);
          krow[i] = k;
          rows[2 * i] = p0 ? k : -1;
          rows[2 * i + 1] = p1 ? K + k : -1;
        }
        n += __popc(bal);
      }
      n *= 2;
    }
    if (lane == 0) s_nrows = n;
  }
  __syncthreads();
  // the crop's rows split evenly over as many groups of at most ROWS as it needs
  // (17 rows: 9 + 8, not 16 + 1); decode mode keeps the slot pairs together
  const int nrows = s_nrows;
  const int ngroups = (nrows + ROWS - 1) / ROWS;
  if (rg >= ngroups) return;
  const int per = decode ? 2 * ((nrows / 2 + ngroups - 1) / ngroups) : (nrows + ngroups - 1) / ngroups;
  const int r0 = rg * per;
  if (r0 >= nrows) return;
  const int nr = min(per, nrows - r0);

  const int px = threadIdx.x % kF32Pix, qc = threadIdx.x / kF32Pix;   // pixel, channel quarter
  const int Y = 4 * band + (px >> 5);
  const int X = 32 * cb + (px & 31);
  int y0, y1, x0, x1;
  float ly, lx;
  taps_f32(Y, h, y0, y1, ly);
  taps_f32(min(X, W - 1), w, x0, x1, lx);
  const float w00 = (1.f - ly) * (1.f - lx), w01 = (1.f - ly) * lx, w10 = ly * (1.f - lx), w11 = ly * lx;
  // the tile's source patch: rows sy0 .. sy0 + 2, columns sx0 .. sx0 + 9 (clamped
  // at the far edges); every tap of the tile falls inside it
  const int sy0 = max(band - 1, 0), sx0 = max(8 * cb - 1, 0);
  const int l00 = ((y0 - sy0) * kPatchCols + (x0 - sx0)) * kLinePitch;
  const int l01 = ((y0 - sy0) * kPatchCols + (x1 - sx0)) * kLinePitch;
  const int l10 = ((y1 - sy0) * kPatchCols + (x0 - sx0)) * kLinePitch;
  const int l11 = ((y1 - sy0) * kPatchCols + (x1 - sx0)) * kLinePitch;
  const float* Fb = feat + static_cast<long long>(b) * h * w * C;
  const float* kb = kern + static_cast<long long>(b) * kern_bs;

  const int nchunk = (C + kF32Chunk - 1) / kF32Chunk;
  const int nround = (nchunk + kF32Quarters - 1) / kF32Quarters;
  // one round's copies, spread over all threads: 4 x 30 patch lines x 8 float4,
  // then 4 x ROWS rows x 8 float4 (zero-filled past C and for absent slots)
  auto issue = [&](int rd, F32Buf<ROWS>& bf) {
    constexpr int kPatchCopies = kF32Quarters * kPatchLines * (kF32Chunk / 4);
    constexpr int kRowCopies = kF32Quarters * ROWS * (kF32Chunk / 4);
    for (int t = threadIdx.x; t < kPatchCopies + kRowCopies; t += kF32Threads) {
      if (t < kPatchCopies) {
        const int qq = t / (kPatchLines * 8), rem = t % (kPatchLines * 8);
        const int line = rem >> 3, f4 = rem & 7;
        const int c = (rd * kF32Quarters + qq) * kF32Chunk + 4 * f4;
        const int y = min(sy0 + line / kPatchCols, h - 1), x = min(sx0 + line % kPatchCols, w - 1);
        const bool full = c < C;
        cp_async16(&bf.patch[qq][line * kLinePitch + 4 * f4],
                   full ? Fb + (static_cast<long long>(y) * w + x) * C + c : Fb, full);
      } else {
        const int u = t - kPatchCopies;
        const int qq = u / (ROWS * 8), rem = u % (ROWS * 8);
        const int r = rem >> 3, f4 = rem & 7;
        const int c = (rd * kF32Quarters + qq) * kF32Chunk + 4 * f4;
        const bool full = r < nr && c < C && rows[r0 + r] >= 0;
        cp_async16(&bf.ks[qq][r][f4], full ? kb + static_cast<long long>(rows[r0 + r]) * C + c : kb, full);
      }
    }
    cp_async_commit();
  };

  float acc[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) acc[r] = 0.f;

  if (nround > 0) issue(0, buf[0]);
  for (int rd = 0; rd < nround; ++rd) {
    if (rd + 1 < nround) {
      issue(rd + 1, buf[(rd + 1) & 1]);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const F32Buf<ROWS>& bf = buf[rd & 1];
    const float* pt = bf.patch[qc];
    // this pixel's upsampled channels of the quarter's chunk
    float u[kF32Chunk];
#pragma unroll
    for (int q = 0; q < kF32Chunk / 4; ++q) {
      const float4 a = *reinterpret_cast<const float4*>(pt + l00 + 4 * q);
      const float4 bq = *reinterpret_cast<const float4*>(pt + l01 + 4 * q);
      const float4 cq = *reinterpret_cast<const float4*>(pt + l10 + 4 * q);
      const float4 dq = *reinterpret_cast<const float4*>(pt + l11 + 4 * q);
      u[4 * q + 0] = fmaf(w11, dq.x, fmaf(w10, cq.x, fmaf(w01, bq.x, w00 * a.x)));
      u[4 * q + 1] = fmaf(w11, dq.y, fmaf(w10, cq.y, fmaf(w01, bq.y, w00 * a.y)));
      u[4 * q + 2] = fmaf(w11, dq.z, fmaf(w10, cq.z, fmaf(w01, bq.z, w00 * a.z)));
      u[4 * q + 3] = fmaf(w11, dq.w, fmaf(w10, cq.w, fmaf(w01, bq.w, w00 * a.w)));
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      if (r < nr) {
        float s = acc[r];
#pragma unroll
        for (int q = 0; q < kF32Chunk / 4; ++q) {
          const float4 kv = bf.ks[qc][r][q];
          s = fmaf(u[4 * q + 0], kv.x, s);
          s = fmaf(u[4 * q + 1], kv.y, s);
          s = fmaf(u[4 * q + 2], kv.z, s);
          s = fmaf(u[4 * q + 3], kv.w, s);
        }
        acc[r] = s;
      }
    }
    __syncthreads();   // the buffer is refilled by the copies issued next round
  }
  // quarter 0 adds the other quarters' partial sums, in quarter order
  if (qc > 0) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
      if (r < nr) red[qc - 1][r][px] = acc[r];
  }
  __syncthreads();
  if (qc > 0) return;
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
    if (r < nr) acc[r] = (acc[r] + red[0][r][px]) + (red[1][r][px] + red[2][r][px]);

  if (decode) {
    // fuse the two modality slots of each prompt row, then one key per row and warp
    const bool inside = Y < H && X < W;
    const uint32_t pixel = inside ? static_cast<uint32_t>(Y * W + X) : 0u;
    const int lane = threadIdx.x & 31;
    unsigned long long mine = 0;
#pragma unroll
    for (int i = 0; i < ROWS / 2; ++i) {
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
    for (int r = 0; r < ROWS; ++r)
      if (r < nr) hb[static_cast<long long>(rows[r0 + r]) * P] = acc[r];
  }
}

template <int ROWS>
static cudaError_t launch_f32_rows(const float* feat, int B, int h, int w, int C, const float* kern,
                                   long long kern_batch_stride, const uint8_t* mask, long long mask_batch_stride,
                                   int M, int K, float* heat, unsigned long long* keys, cudaStream_t stream) {
  const int W = 4 * w;
  const int groups = keys ? (K + ROWS / 2 - 1) / (ROWS / 2) : (M * K + ROWS - 1) / ROWS;
  dim3 grid(h * ((W + 31) / 32), groups, B);
  const size_t smem = f32_smem_bytes<ROWS>();
  cudaError_t e = cudaFuncSetAttribute(heatmap_f32_kernel<ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  heatmap_f32_kernel<ROWS><<<grid, kF32Threads, smem, stream>>>(feat, h, w, C, kern, kern_batch_stride, mask,
                                                              mask_batch_stride, M, K, heat, keys);
  return cudaGetLastError();
}

cudaError_t launch_heatmap_f32(const float* feat, int B, int h, int w, int C, const float* kern,
                               long long kern_batch_stride, const uint8_t* mask, long long mask_batch_stride, int M,
                               int K, float* heat, unsigned long long* keys, int num_sms, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  const long long tiles = static_cast<long long>(B) * h * ((4 * w + 31) / 32);
  if (tiles >= 2LL * num_sms)
    return launch_f32_rows<32>(feat, B, h, w, C, kern, kern_batch_stride, mask, mask_batch_stride, M, K, heat, keys,
                               stream);
  return launch_f32_rows<16>(feat, B, h, w, C, kern, kern_batch_stride, mask, mask_batch_stride, M, K, heat, keys,
                             stream);
}

}  // namespace gkd
