// Steps a3 + a4 on the tensor cores: bilinear 4x upsample (align_corners=False)
// of the query feature map fused into the operand staging of the 1x1
// dynamic-kernel contraction heat[b,m,k,p] = sum_c khat[b,m,k,c] * U[b,p,c]
// ("bilinear 4x upsample ... 1x1 kernel conv", GKD_GGUF model card, "Model"
// section, Architecture bullet; "kernels convolve over the query image's
// features", GKDT summary page, pipeline paragraph).
//
// GEMM view per crop: D[pixel, row] = U[pixel, :] . khat[row, :], M = pixels,
// N = the crop's valid prompt rows, K = channels. Operands are bf16, the sum is
// fp32 in tensor memory.
//
// Persistent kernel, one CTA per SM, 14 warps:
//   warp 0      TMA: per 64-channel chunk, a 3x10-patch feature slab (128B
//               swizzled) and the crop's kernel-row segments (the B operand);
//   warp 1      MMA issuer: tcgen05.mma kind::f16, A from TMEM, B from smem;
//   warps 2-5   epilogue: tcgen05.ld of the accumulators, heatmap stores;
//   warps 6-13  upsample producers: each thread owns a vertical pixel pair
//               sharing the same four source taps, lerps in fp32 (packed f32x2),
//               rounds to bf16 and writes the A operand straight into TMEM with
//               tcgen05.st (never through shared memory).
// A work unit is 8 output rows x 32 output columns (256 pixels = two M=128
// tiles that share the B operand). Units are split over CTAs by a static
// cost-balanced partition computed in the prologue. Every wait is bounded; a
// timeout sets the device error word and all roles drain and exit.
#include <cstdio>

#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {
namespace tc {

constexpr int kStages = 3;
constexpr int kChunk = 64;                       // channels per K-chunk
constexpr int kMaxN = 160;                       // accumulator columns per tile
constexpr int kUnitRows = 8, kUnitCols = 32;
constexpr int kSlabRows = 3, kSlabCols = 10;
constexpr int kSlabHalf = 4096;                  // 30 lines x 128 B, padded to 1 KB multiple
constexpr int kSlabBytes = 2 * kSlabHalf;
constexpr int kBBytes = kMaxN * 128;
constexpr int kStageBytes = kSlabBytes + kBBytes;  // 28 KB, 1 KB aligned
constexpr int kNumWarps = 14, kThreads = kNumWarps * 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpProd0 = 6;   // warps 2-5: epilogue
constexpr int kNumProdWarps = 8, kNumEpiWarps = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColD0 = 0, kColD1 = kMaxN, kColA = 2 * kMaxN;   // A stages at 320, 384, 448
constexpr int kCostBias = 48;                    // per-unit cost model: N + bias
constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + 256 + 32 * 1024;  // padded: one CTA per SM

struct Smem {            // control block placed after the stage buffers
  uint64_t full[kStages];
  uint64_t afull[kStages];
  uint64_t empty[kStages];
  uint64_t accfull;
  uint64_t accempty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  unsigned long long unit_begin, unit_end;
  long long total_cost;
};

struct CropInfo {
  int n;                 // accumulator columns (multiple of 16), 0 = nothing to do
  int kmin[2], len[2], off[2];
  uint32_t vbits[5];     // bit c of word c/32: column c maps to a valid (m, k) row
};

__device__ __forceinline__ const uint8_t* crop_mask(const HeatmapTcArgs& a, int b) {
  return a.mask + static_cast<long long>(b) * a.mask_batch_stride;
}

// Warp-cooperative: valid-row segments of one crop (all lanes get the result).
__device__ __forceinline__ CropInfo crop_info(const HeatmapTcArgs& a, int b, int lane) {
  CropInfo ci;
  const uint8_t* mb = crop_mask(a, b);
  int off = 0;
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    ci.kmin[m] = 0;
    ci.len[m] = 0;
    ci.off[m] = off;
    if (m >= a.M) continue;
    int first = a.K, last = -1;
    for (int kb = 0; kb < a.K; kb += 32) {
      const int k = kb + lane;
      const bool v = (k < a.K) && mb[m * a.K + k] != 0;
      const unsigned bal = __ballot_sync(0xffffffffu, v);
      if (bal) {
        first = min(first, kb + __ffs(bal) - 1);
        last = kb + 31 - __clz(bal);
      }
    }
    if (last >= 0) {
      ci.kmin[m] = first;
      ci.len[m] = (last - first + 1 + 7) & ~7;
      off += ci.len[m];
    }
  }
  ci.n = (off + 15) & ~15;
#pragma unroll
  for (int g = 0; g < 5; ++g) {
    const int col = g * 32 + lane;
    bool v = false;
    if (col < off) {
      const int m = (a.M == 2 && col >= ci.off[1]) ? 1 : 0;
      const int k = ci.kmin[m] + (col - ci.off[m]);
      v = (col - ci.off[m] < ci.len[m]) && k < a.K && mb[m * a.K + k] != 0;
    }
    ci.vbits[g] = __ballot_sync(0xffffffffu, v);
  }
  return ci;
}

// Thread-local (no warp collectives): number of accumulator columns of a crop.
__device__ __forceinline__ int crop_n_serial(const HeatmapTcArgs& a, int b) {
  const uint8_t* mb = crop_mask(a, b);
  int off = 0;
  for (int m = 0; m < a.M; ++m) {
    int first = -1, last = -1;
    for (int k = 0; k < a.K; ++k)
      if (mb[m * a.K + k]) {
        if (first < 0) first = k;
        last = k;
      }
    if (last >= 0) off += (last - first + 1 + 7) & ~7;
  }
  return (off + 15) & ~15;
}

__device__ __forceinline__ void src_taps(int d, int n, int& i0, int& i1, float& lam) {
  const float s = fmaxf((static_cast<float>(d) + 0.5f) * 0.25f - 0.5f, 0.0f);
  i0 = static_cast<int>(s);
  i1 = min(i0 + 1, n - 1);
  lam = s - static_cast<float>(i0);
}

__device__ __forceinline__ uint32_t make_idesc(int n) {
  // kind::f16: D fp32 (bit 4), A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 = 1),
  // both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28 (M = 128).
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ uint64_t make_bdesc(uint32_t smem_addr) {
  // K-major, 128B swizzle: LBO = 1 (16 B), SBO = 1024 B (8 rows x 128 B), version 1, layout 2.
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void set_abort(Smem* ctl, unsigned* err, unsigned bits) {
  ctl->abort_flag = 1;
  atomicOr(err, bits);
}

__device__ __forceinline__ float2 f2sub(float2 b, float2 a) {   // b - a, one rounding
  return __ffma2_rn(a, make_float2(-1.f, -1.f), b);
}

struct PixelPair {
  int Ya, X;        // upper pixel; the lower one is (Ya + 1, X)
  int L00, L01, L10, L11;   // slab lines of the four taps
  float2 lx, la, lb;        // lerp weights (broadcast to both lanes of a float2)
};

__device__ __forceinline__ PixelPair pair_geometry(const HeatmapTcArgs& a, int vb, int ub, int q, int lane) {
  PixelPair pp;
  const int Y0 = kUnitRows * vb - 2, X0 = kUnitCols * ub;
  const int Yg = Y0 + ((q >> 1) << 2);
  pp.Ya = Yg + 2 * (lane >> 4);
  pp.X = X0 + ((q & 1) << 4) + (lane & 15);
  int r0, r1, r0b, r1b, c0, c1;
  float lya, lyb, lxx;
  src_taps(pp.Ya, a.h, r0, r1, lya);
  src_taps(pp.Ya + 1, a.h, r0b, r1b, lyb);
  src_taps(pp.X, a.w, c0, c1, lxx);
  // both pixels of the pair read the same two source rows (r0, r1)
  const int sr0 = r0 - (2 * vb - 1), sr1 = r1 - (2 * vb - 1);
  const int sc0 = c0 - (8 * ub - 1), sc1 = c1 - (8 * ub - 1);
  pp.L00 = sr0 * kSlabCols + sc0;
  pp.L01 = sr0 * kSlabCols + sc1;
  pp.L10 = sr1 * kSlabCols + sc0;
  pp.L11 = sr1 * kSlabCols + sc1;
  pp.lx = make_float2(lxx, lxx);
  pp.la = make_float2(lya, lya);
  pp.lb = make_float2(lyb, lyb);
  return pp;
}

__device__ __forceinline__ const uint8_t* swz(const uint8_t* base, int line, int chunk16) {
  return base + line * 128 + (((chunk16 ^ (line & 7))) << 4);
}

// Upsample two fp32 channel pairs of a pixel pair; writes packed bf16x2 words.
__device__ __forceinline__ void lerp_pair(float2 f00, float2 f01, float2 f10, float2 f11, const PixelPair& pp,
                                          uint32_t& oa, uint32_t& ob) {
  const float2 t0 = __ffma2_rn(pp.lx, f2sub(f01, f00), f00);
  const float2 t1 = __ffma2_rn(pp.lx, f2sub(f11, f10), f10);
  const float2 dt = f2sub(t1, t0);
  const float2 ua = __ffma2_rn(pp.la, dt, t0);
  const float2 ubv = __ffma2_rn(pp.lb, dt, t0);
  oa = pack_bf16x2(ua.x, ua.y);
  ob = pack_bf16x2(ubv.x, ubv.y);
}

__device__ __forceinline__ float2 bf16lo_hi(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) heatmap_tc_kernel(const __grid_constant__ HeatmapTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem* ctl = reinterpret_cast<Smem*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  const int H = 4 * a.h, W = 4 * a.w;
  const int nbands = (H + 2 + kUnitRows - 1) / kUnitRows;
  const int ncb = (W + kUnitCols - 1) / kUnitCols;
  const long long nU = static_cast<long long>(nbands) * ncb;
  const int nchunks = (a.C + kChunk - 1) / kChunk;
  const long long P = static_cast<long long>(H) * W;

  // ---------------- prologue: barriers, TMEM, work partition ----------------
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->afull[s], kNumProdWarps);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->accfull, 1);
    mbar_init(&ctl->accempty, kNumEpiWarps);
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    ctl->unit_begin = ~0ull;
    ctl->unit_end = ~0ull;
    ctl->total_cost = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&a.tmap_feat);
    tma_prefetch_desc(&a.tmap_kern8);
    tma_prefetch_desc(&a.tmap_kern32);
  }
  __syncthreads();

  const long long G = gridDim.x, g = blockIdx.x;
  const unsigned long long total_units = static_cast<unsigned long long>(a.B) * nU;
  if (a.kern_shared && a.mask_batch_stride == 0) {
    // every crop has the same rows: split the units evenly
    if (tid == 0) {
      const int n0 = crop_n_serial(a, 0);
      if (n0 == 0) {
        ctl->unit_begin = ctl->unit_end = 0;
      } else {
        ctl->unit_begin = (total_units * g + G - 1) / G;
        ctl->unit_end = (total_units * (g + 1) + G - 1) / G;
      }
    }
  } else {
    // pass 1: total cost
    long long local = 0;
    for (int b = tid; b < a.B; b += kThreads) {
      const int n = crop_n_serial(a, b);
      if (n) local += (n + kCostBias) * nU;
    }
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if (lane == 0 && local) atomicAdd(reinterpret_cast<unsigned long long*>(&ctl->total_cost),
                                      static_cast<unsigned long long>(local));
    __syncthreads();
    const long long T = ctl->total_cost;
    const long long tgt0 = g * T, tgt1 = (g + 1) * T;
    // pass 2: first unit whose cumulative cost before it reaches g*T/G (resp. (g+1)*T/G)
    __shared__ long long s_scan[kNumWarps];
    long long carry = 0;
    for (int base = 0; base < a.B; base += kThreads) {
      const int b = base + tid;
      const int n = (b < a.B) ? crop_n_serial(a, b) : 0;
      const long long c = n ? (n + kCostBias) : 0;
      const long long tot = c * nU;
      long long incl = tot;
      for (int o = 1; o < 32; o <<= 1) {
        const long long v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) s_scan[warp] = incl;
      __syncthreads();
      long long wbase = 0, btot = 0;
      for (int w2 = 0; w2 < kNumWarps; ++w2) {
        if (w2 < warp) wbase += s_scan[w2];
        btot += s_scan[w2];
      }
      const long long cb = carry + wbase + incl - tot;
      if (c > 0) {
        const long long cg = c * G;
        long long need = tgt0 - cb * G;
        long long j = need <= 0 ? 0 : (need + cg - 1) / cg;
        if (j < nU) atomicMin(&ctl->unit_begin, static_cast<unsigned long long>(b) * nU + j);
        need = tgt1 - cb * G;
        j = need <= 0 ? 0 : (need + cg - 1) / cg;
        if (j < nU) atomicMin(&ctl->unit_end, static_cast<unsigned long long>(b) * nU + j);
      }
      carry += btot;
      __syncthreads();
    }
    if (tid == 0) {
      if (ctl->unit_begin == ~0ull) ctl->unit_begin = total_units;
      if (ctl->unit_end == ~0ull) ctl->unit_end = total_units;
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const unsigned long long ubeg = ctl->unit_begin, uend = ctl->unit_end;
  const uint64_t lim = a.wait_limit_ns;
  volatile int* abortp = &ctl->abort_flag;

  if (warp == kWarpTma) {
    // ---------------------------------------------------------------- TMA
    uint32_t it = 0;
    int cur_b = -1;
    CropInfo ci{};
    bool ok = true;
    for (unsigned long long u = ubeg; u < uend && ok; ++u) {
      const int b = static_cast<int>(u / nU), j = static_cast<int>(u % nU);
      if (b != cur_b) { ci = crop_info(a, b, lane); cur_b = b; }
      if (ci.n == 0) continue;
      const int vb = j / ncb, ub = j % ncb;
      const int bk = a.kern_shared ? 0 : b;
      for (int ch = 0; ch < nchunks; ++ch, ++it) {
        const int s = it % kStages;
        const uint32_t use = it / kStages;
        if (use > 0 && !mbar_wait_bounded(&ctl->empty[s], (use & 1) ^ 1, lim, abortp)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t bytes = (a.feat_bf16 ? kSlabRows * kSlabCols * 128 : 2 * kSlabRows * kSlabCols * 128) +
                                 (ci.len[0] + ci.len[1]) * 128;
          mbar_arrive_expect_tx(&ctl->full[s], bytes);
          const int c0 = ch * kChunk;
          if (a.feat_bf16) {
            tma_load_4d(st, &a.tmap_feat, &ctl->full[s], c0, 8 * ub - 1, 2 * vb - 1, b);
          } else {
            tma_load_4d(st, &a.tmap_feat, &ctl->full[s], c0, 8 * ub - 1, 2 * vb - 1, b);
            tma_load_4d(st + kSlabHalf, &a.tmap_feat, &ctl->full[s], c0 + 32, 8 * ub - 1, 2 * vb - 1, b);
          }
          uint8_t* bdst = st + kSlabBytes;
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int len = ci.len[m], off = ci.off[m], kmin = ci.kmin[m];
            int r = 0;
            for (; len - r >= 32; r += 32)
              tma_load_4d(bdst + (off + r) * 128, &a.tmap_kern32, &ctl->full[s], c0, kmin + r, m, bk);
            for (; r < len; r += 8)
              tma_load_4d(bdst + (off + r) * 128, &a.tmap_kern8, &ctl->full[s], c0, kmin + r, m, bk);
          }
        }
        __syncwarp();
      }
    }
    // drain: make sure no load issued by this warp is still landing in shared memory
    if (lane == 0) {
      for (uint32_t k = 0; k < kStages && k < it; ++k) {
        const uint32_t last = it - 1 - k;
        if (!mbar_wait_drain(&ctl->full[last % kStages], (last / kStages) & 1, lim)) atomicOr(a.err, kErrTimeout);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    uint32_t it = 0, v = 0;
    int cur_b = -1;
    CropInfo ci{};
    bool ok = true;
    for (unsigned long long u = ubeg; u < uend && ok; ++u) {
      const int b = static_cast<int>(u / nU);
      if (b != cur_b) { ci = crop_info(a, b, lane); cur_b = b; }
      if (ci.n == 0) continue;
      const uint32_t idesc = make_idesc(ci.n);
      if (v > 0 && !mbar_wait_bounded(&ctl->accempty, (v - 1) & 1, lim, abortp)) {
        if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
        ok = false;
        break;
      }
      tc_fence_after();
      for (int ch = 0; ch < nchunks; ++ch, ++it) {
        const int s = it % kStages;
        const uint32_t par = (it / kStages) & 1;
        if (!mbar_wait_bounded(&ctl->full[s], par, lim, abortp) ||
            !mbar_wait_bounded(&ctl->afull[s], par, lim, abortp)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t bbase = smem_u32(smem + s * kStageBytes + kSlabBytes);
          const uint32_t acol = kColA + s * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = make_bdesc(bbase + kk * 32);
            const uint32_t acc = (ch > 0 || kk > 0) ? 1u : 0u;
            umma_ts_f16(tmem + kColD0, tmem + acol + kk * 8, bd, idesc, acc);
            umma_ts_f16(tmem + kColD1, tmem + acol + 32 + kk * 8, bd, idesc, acc);
          }
          umma_commit(&ctl->empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&ctl->accfull);
      __syncwarp();
      ++v;
    }
    // drain: wait until every MMA issued by this thread has completed
    if (lane == 0 && it > 0) {
      umma_commit(&ctl->drain);
      if (!mbar_wait_drain(&ctl->drain, 0, lim)) atomicOr(a.err, kErrTimeout);
    }
    __syncwarp();
  } else if (warp < kWarpProd0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    uint32_t v = 0;
    int cur_b = -1;
    CropInfo ci{};
    for (unsigned long long u = ubeg; u < uend; ++u) {
      const int b = static_cast<int>(u / nU), j = static_cast<int>(u % nU);
      if (b != cur_b) { ci = crop_info(a, b, lane); cur_b = b; }
      if (ci.n == 0) continue;
      if (!mbar_wait_bounded(&ctl->accfull, v & 1, lim, abortp)) {
        if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const PixelPair pp = pair_geometry(a, j / ncb, j % ncb, q, lane);
      const bool xin = pp.X < W;
      const bool ya_in = pp.Ya >= 0 && pp.Ya < H, yb_in = pp.Ya + 1 >= 0 && pp.Ya + 1 < H;
      float* hb = a.heat + static_cast<long long>(b) * a.M * a.K * P;
      const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
      for (int n0 = 0; n0 < ci.n; n0 += 16) {
        uint32_t word = ci.vbits[0];
#pragma unroll
        for (int g2 = 1; g2 < 5; ++g2)
          if ((n0 >> 5) == g2) word = ci.vbits[g2];
        const uint32_t bits16 = (word >> (n0 & 31)) & 0xFFFFu;
        if (bits16 == 0) continue;
        uint32_t v0[16], v1[16];
        tmem_ld_32x32b_x16(tmem + lane_off + kColD0 + n0, v0);
        tmem_ld_32x32b_x16(tmem + lane_off + kColD1 + n0, v1);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int col = n0 + jj;
          if (!((bits16 >> jj) & 1u)) continue;
          const bool m1 = a.M == 2 && col >= ci.off[1];
          const int m = m1 ? 1 : 0;
          const int k = (m1 ? ci.kmin[1] : ci.kmin[0]) + (col - (m1 ? ci.off[1] : 0));
          float* row = hb + (static_cast<long long>(m) * a.K + k) * P;
          if (xin) {
            if (ya_in) __stcs(row + static_cast<long long>(pp.Ya) * W + pp.X, __uint_as_float(v0[jj]));
            if (yb_in) __stcs(row + static_cast<long long>(pp.Ya + 1) * W + pp.X, __uint_as_float(v1[jj]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->accempty);
      ++v;
    }
  } else {
    // ---------------------------------------------------------------- upsample producers
    const int q = warp & 3;
    const int hsel = (warp - kWarpProd0) >> 2;   // which 32 channels of each chunk
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const bool skip_first = (a.debug_flags & kDbgSkipProducerArrive) != 0;
    uint32_t it = 0;
    int cur_b = -1;
    CropInfo ci{};
    bool ok = true;
    for (unsigned long long u = ubeg; u < uend && ok; ++u) {
      const int b = static_cast<int>(u / nU), j = static_cast<int>(u % nU);
      if (b != cur_b) { ci = crop_info(a, b, lane); cur_b = b; }
      if (ci.n == 0) continue;
      const PixelPair pp = pair_geometry(a, j / ncb, j % ncb, q, lane);
      for (int ch = 0; ch < nchunks; ++ch, ++it) {
        const int s = it % kStages;
        const uint32_t use = it / kStages;
        if (!mbar_wait_bounded(&ctl->full[s], use & 1, lim, abortp) ||
            (use > 0 && !mbar_wait_bounded(&ctl->empty[s], (use & 1) ^ 1, lim, abortp))) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* slab = smem + s * kStageBytes;
        const uint32_t acol = tmem + lane_off + kColA + s * 64 + hsel * 16;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {      // two halves of 16 channels: 8 TMEM columns each
          uint32_t oa[8], ob[8];
          if (!a.feat_bf16) {
            const uint8_t* half = slab + hsel * kSlabHalf;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int g4 = hh * 4 + g;
              const float4 f00 = *reinterpret_cast<const float4*>(swz(half, pp.L00, g4));
              const float4 f01 = *reinterpret_cast<const float4*>(swz(half, pp.L01, g4));
              const float4 f10 = *reinterpret_cast<const float4*>(swz(half, pp.L10, g4));
              const float4 f11 = *reinterpret_cast<const float4*>(swz(half, pp.L11, g4));
              lerp_pair(make_float2(f00.x, f00.y), make_float2(f01.x, f01.y), make_float2(f10.x, f10.y),
                        make_float2(f11.x, f11.y), pp, oa[2 * g], ob[2 * g]);
              lerp_pair(make_float2(f00.z, f00.w), make_float2(f01.z, f01.w), make_float2(f10.z, f10.w),
                        make_float2(f11.z, f11.w), pp, oa[2 * g + 1], ob[2 * g + 1]);
            }
          } else {
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int chunk = hsel * 4 + hh * 2 + g;
              const uint4 u00 = *reinterpret_cast<const uint4*>(swz(slab, pp.L00, chunk));
              const uint4 u01 = *reinterpret_cast<const uint4*>(swz(slab, pp.L01, chunk));
              const uint4 u10 = *reinterpret_cast<const uint4*>(swz(slab, pp.L10, chunk));
              const uint4 u11 = *reinterpret_cast<const uint4*>(swz(slab, pp.L11, chunk));
              lerp_pair(bf16lo_hi(u00.x), bf16lo_hi(u01.x), bf16lo_hi(u10.x), bf16lo_hi(u11.x), pp,
                        oa[4 * g + 0], ob[4 * g + 0]);
              lerp_pair(bf16lo_hi(u00.y), bf16lo_hi(u01.y), bf16lo_hi(u10.y), bf16lo_hi(u11.y), pp,
                        oa[4 * g + 1], ob[4 * g + 1]);
              lerp_pair(bf16lo_hi(u00.z), bf16lo_hi(u01.z), bf16lo_hi(u10.z), bf16lo_hi(u11.z), pp,
                        oa[4 * g + 2], ob[4 * g + 2]);
              lerp_pair(bf16lo_hi(u00.w), bf16lo_hi(u01.w), bf16lo_hi(u10.w), bf16lo_hi(u11.w), pp,
                        oa[4 * g + 3], ob[4 * g + 3]);
            }
          }
          tmem_st_32x32b_x8(acol + hh * 8, oa);
          tmem_st_32x32b_x8(acol + 32 + hh * 8, ob);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && !(skip_first && it == 0)) mbar_arrive(&ctl->afull[s]);
      }
    }
    tmem_wait_st();
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc

static bool encode(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, const void* base,
                   const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_heatmap_tc(HeatmapTcArgs& a, const void* feat, const void* kern, long long kern_batch_stride,
                              int num_sms, cudaStream_t stream, const char** why) {
  if (a.B == 0) return cudaSuccess;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) {
    *why = "cuTensorMapEncodeTiled is unavailable";
    return cudaErrorNotSupported;
  }
  const cuuint64_t C = a.C, w = a.w, h = a.h, B = a.B;
  if (a.feat_bf16) {
    const cuuint64_t dims[4] = {C, w, h, B};
    const cuuint64_t strides[3] = {C * 2, w * C * 2, h * w * C * 2};
    const cuuint32_t box[4] = {64, tc::kSlabCols, tc::kSlabRows, 1};
    if (!encode(enc, &a.tmap_feat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, feat, dims, strides, box)) {
      *why = "tensor map encoding failed for the bf16 feature map";
      return cudaErrorInvalidValue;
    }
  } else {
    const cuuint64_t dims[4] = {C, w, h, B};
    const cuuint64_t strides[3] = {C * 4, w * C * 4, h * w * C * 4};
    const cuuint32_t box[4] = {32, tc::kSlabCols, tc::kSlabRows, 1};
    if (!encode(enc, &a.tmap_feat, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, feat, dims, strides, box)) {
      *why = "tensor map encoding failed for the fp32 feature map";
      return cudaErrorInvalidValue;
    }
  }
  {
    const cuuint64_t Bk = a.kern_shared ? 1 : static_cast<cuuint64_t>(a.B);
    const cuuint64_t K = a.K, M = a.M;
    const cuuint64_t bstride = a.kern_shared ? M * K * C * 2 : static_cast<cuuint64_t>(kern_batch_stride) * 2;
    const cuuint64_t dims[4] = {C, K, M, Bk};
    const cuuint64_t strides[3] = {C * 2, K * C * 2, bstride};
    const cuuint32_t box8[4] = {64, 8, 1, 1};
    const cuuint32_t box32[4] = {64, 32, 1, 1};
    if (!encode(enc, &a.tmap_kern8, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kern, dims, strides, box8) ||
        !encode(enc, &a.tmap_kern32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kern, dims, strides, box32)) {
      *why = "tensor map encoding failed for the kernel rows";
      return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(tc::heatmap_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(tc::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int H = 4 * a.h, W = 4 * a.w;
  const long long nU = static_cast<long long>((H + 2 + tc::kUnitRows - 1) / tc::kUnitRows) *
                       ((W + tc::kUnitCols - 1) / tc::kUnitCols);
  const long long units = nU * a.B;
  const int grid = static_cast<int>(units < num_sms ? units : num_sms);
  tc::heatmap_tc_kernel<<<grid, tc::kThreads, tc::kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gkd
