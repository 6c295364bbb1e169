// Steps a3 + a4 on the tensor cores: bilinear 4x upsample (align_corners=False)
// of the query feature map fused into the operand staging of the 1x1
// dynamic-kernel contraction heat[b,m,k,p] = sum_c khat[b,m,k,c] * U[b,p,c]
// (4x bilinear upsample and prompts applied as 1x1 convolution kernels: GKD_GGUF
// model card, Model section, Architecture bullet; the prompt kernels are
// convolved over the query features: GKDT summary page, pipeline paragraph).
//
// GEMM view per crop: D[pixel, row] = U[pixel, :] . khat[row, :], M = pixels,
// N = the crop's valid prompt rows, K = channels. Operands are bf16, the sum is
// fp32 in tensor memory.
//
// One CTA per SM (218 KB of shared memory, all 512 tensor-memory columns), 24
// warps, one M=128 tile (4 output rows x 32 output columns, which all read the
// same two source rows) per work unit:
//   warp 0       TMA: per 128-channel stage, a 2x10-patch feature slab (128B
//                swizzled) into a 6-deep ring; warp 1: TMA of the stage's
//                kernel rows (the B operand, one box per modality) into a 3-deep ring;
//   warp 2       MMA issuer: tcgen05.mma kind::f16 issued by one elected lane,
//                A from tensor memory, B from shared memory, into one of two
//                accumulator buffers, so the next unit accumulates while the
//                epilogue drains;
//   warps 3-10   epilogue, two sets of four (one warp per tensor-memory lane
//                quadrant) taking alternate 16-column groups: tcgen05.ld of the
//                accumulator, transpose through a padded shared tile, coalesced
//                float4 heatmap rows;
//   warps 11-22  upsample producers in three groups of four warps (one warp per
//                lane quadrant); group g builds the A operand of every stage i
//                with i % 3 == g, so each warp has three stage periods for its
//                own. A thread owns one output column of four pixels (one x-lerp
//                per source row serves all four) and 32 channels of the stage,
//                lerps in fp32 (packed f32x2), rounds to bf16 and writes the A
//                operand straight into tensor memory;
//   warp 23      unit scheduler: the grid has one CTA per unit; a running CTA
//                does its own unit, then takes over the units of CTAs that have
//                not started yet with cluster launch control (a cancelled CTA
//                never runs), so the SMs balance the work among themselves as
//                they go. It publishes each unit with its crop's row segments
//                into an 8-slot ring that every other warp reads.
// Every wait is bounded, and every role takes the outcome of a wait as one
// decision for all of its threads; a timeout sets the device error word and all
// roles drain their in-flight copies and MMAs and exit.
#include "decode_key.cuh"
#include "gkd_internal.h"
#include "ptx.cuh"

namespace gkd {
namespace tc {

// Optional timeline tracing (build with -DGKD_TRACE): CTA 0 records %globaltimer
// at each hand-off between roles; read back with gkd_trace_read().
#ifdef GKD_TRACE
__device__ unsigned long long g_trace[16][2048];
__device__ unsigned long long g_cta[1024][4];     // per CTA: start, end (ns), units, sum of n
__device__ unsigned long long g_entry[1024];      // per CTA: kernel entry (ns)
#define GKD_TR(kind, idx) \
  do { if (blockIdx.x == 0 && (idx) < 2048u) g_trace[kind][idx] = global_timer_ns(); } while (0)
#else
#define GKD_TR(kind, idx) do { } while (0)
#endif

constexpr int kSlabStages = 6;                   // slab ring (smem), freed by the producers
constexpr int kStages = 3;                       // kernel rows (smem) + A operand (tmem), freed by the MMA
constexpr int kChunk = 128;                      // channels per stage: two 64-channel sub-chunks
constexpr int kSub = 64;                         // channels per A sub-chunk (32 TMEM columns)
constexpr int kMaxN = 160;                       // accumulator columns per tile
constexpr int kUnitRows = 4, kUnitCols = 32;     // one M=128 tile: 4 output rows x 32 output columns
constexpr int kSlabRows = 2, kSlabCols = 10, kSlabLines = kSlabRows * kSlabCols;
constexpr int kPlaneBytes = kSlabLines * 128;    // one 128-byte-wide slab plane (32 fp32 / 64 bf16 channels)
constexpr int kPlaneSplit = 3072;                // plane pitch when each plane is its own box (1 KB aligned)
constexpr int kSlabBytes = 4 * kPlaneSplit;      // fp32: 4 planes; bf16: 2 planes
constexpr int kBSubBytes = kMaxN * 128;          // kernel rows of one sub-chunk
constexpr int kBBytes = 2 * kBSubBytes;          // 40 KB per stage, 1 KB aligned
#ifndef GKD_STORE_REPS
#define GKD_STORE_REPS 1
#endif
constexpr int kStoreReps = GKD_STORE_REPS;       // 16x256b repetitions per producer store (1, 2 or 4)
static_assert(kStoreReps == 1 || kStoreReps == 2 || kStoreReps == 4, "producer store width");
constexpr int kEpiCols = 16;

constexpr int kDecCols = 8;                      // prompt rows per decode-mode block (len is a multiple of 8)                     // accumulator columns per epilogue group
constexpr int kEpiStride = 40;                   // floats per (column, row) line of the epilogue tile
constexpr int kEpiBufBytes = kEpiCols * kUnitRows * kEpiStride * 4;   // 10 KB
// Producer groups take the stages in turn. A group that last built stage i - G
// waits for the MMA to free A slot i % kStages and for slab slot i % kSlabStages
// to fill; a parity wait is unambiguous only if the group itself saw the
// previous phase of both barriers, so G must not exceed kStages and must divide
// kSlabStages.
#ifndef GKD_EPI_HALVES
#define GKD_EPI_HALVES 2
#endif
// Epilogue: kEpiHalves sets of four warps (one per lane quadrant); set e drains
// the accumulator's column groups e, e + kEpiHalves, ...
constexpr int kEpiHalves = GKD_EPI_HALVES;
static_assert(kEpiHalves == 1 || kEpiHalves == 2, "epilogue sets");
#ifndef GKD_PROD_GROUPS
#define GKD_PROD_GROUPS 3
#endif
constexpr int kProdGroups = GKD_PROD_GROUPS, kProdGroupWarps = 4;   // one warp per lane quadrant
constexpr int kNumProdWarps = kProdGroups * kProdGroupWarps, kNumEpiWarps = 4 * kEpiHalves;
constexpr int kNumWarps = 4 + kNumEpiWarps + kNumProdWarps, kThreads = kNumWarps * 32;
constexpr int kWarpTma = 0, kWarpTmaB = 1, kWarpMma = 2, kWarpEpi0 = 3, kWarpProd0 = 3 + kNumEpiWarps;
constexpr int kWarpSched = kNumWarps - 1;        // the unit scheduler (after the producers)
constexpr int kUnitSlots = 8;                    // published units not yet read by every other warp
constexpr int kEpiBarrier = 1;                   // named barriers 1, 2: one per epilogue set of four warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColA = 2 * kMaxN;            // accumulators at 0 and 160; A stages at 320 + 64 s
static_assert(kProdGroups <= kStages && kSlabStages % kProdGroups == 0, "producer groups alias ring phases");
constexpr size_t kCtlBytes = 1024;
constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kSlabStages) * kSlabBytes +
                              static_cast<size_t>(kStages) * kBBytes + 2 * kEpiBufBytes + kCtlBytes;

struct CropInfo {
  int n;                 // accumulator columns (multiple of 16), 0 = nothing to do
  int kmin0, kmin1, len0, len1, off1;
};

struct alignas(16) UnitInfo {   // one work unit as the scheduler publishes it
  int b, j, last, pad0;         // crop, tile within the crop; last: no more units
  CropInfo ci;                  // the crop's row segments
  uint32_t colbits[5];          // bit c of word g: accumulator column 32 g + c holds a valid row
  int pad1;
};
static_assert(sizeof(UnitInfo) == 64, "unit slot size");

struct Smem {            // control block placed after the stage and epilogue buffers
  uint4 clc_resp;              // cluster-launch-control response (16-byte aligned)
  UnitInfo units[kUnitSlots];  // the unit ring
  uint64_t ufull[kUnitSlots];  // unit published (scheduler)
  uint64_t uempty[kUnitSlots]; // unit read by every other warp
  uint64_t clc_bar;            // cancellation response landed
  uint64_t sfull[kSlabStages];
  uint64_t sempty[kSlabStages];
  uint64_t bfull[kStages];     // kernel rows landed (TMA bytes)
  uint64_t ready[kStages];     // A operand written (one arrival per warp of the stage's producer group)
  uint64_t empty[kStages];     // MMA done with kernel rows and A operand
  uint64_t accfull[2];
  uint64_t accempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) <= kCtlBytes, "control block");

__device__ __forceinline__ const uint8_t* crop_mask(const HeatmapTcArgs& a, int b) {
  return a.mask + static_cast<long long>(b) * a.mask_batch_stride;
}

// Warp-cooperative: valid-row segments of one crop (all lanes get the result).
// Segment m covers rows [kmin_m, kmin_m + len_m) of modality m (len a multiple of
// 8) and lands at accumulator columns [off_m, off_m + len_m), off_0 = 0. With
// `aligned` (decode mode) the segments of the modalities present share one row
// range, so the two heatmaps of a prompt row sit exactly off_1 columns apart.
__device__ __forceinline__ CropInfo crop_info(const HeatmapTcArgs& a, int b, int lane, bool aligned) {
  CropInfo ci;
  const uint8_t* mb = crop_mask(a, b);
  // lane l holds mask bytes 8l .. 8l+7 of the crop's [M][K] mask (M K <= 256):
  // eight independent loads, so one memory latency per crop
  const int total = a.M * a.K;
  uint32_t lb = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = 8 * lane + i;
    if (p < total && mb[p] != 0) lb |= 1u << i;
  }
  int kmin[2] = {0, 0}, len[2] = {0, 0}, last_[2] = {-1, -1};
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    if (m >= a.M) continue;
    // this lane's valid positions of modality m, as k indices
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
      kmin[m] = first;
      last_[m] = last;
      len[m] = (last - first + 1 + 7) & ~7;
    }
  }
  if (aligned && last_[0] >= 0 && last_[1] >= 0) {
    const int k0 = min(kmin[0], kmin[1]), k1 = max(last_[0], last_[1]);
    kmin[0] = kmin[1] = k0;
    len[0] = len[1] = (k1 - k0 + 1 + 7) & ~7;
  }
  ci.kmin0 = kmin[0];
  ci.kmin1 = kmin[1];
  ci.len0 = len[0];
  ci.len1 = len[1];
  ci.off1 = len[0];
  const int used = len[0] + len[1];
  ci.n = (used + 15) & ~15;
  return ci;
}

// Warp-cooperative: bit c of word g says accumulator column 32 g + c holds a
// valid (m, k) row of crop b (every lane gets the five words).
__device__ __forceinline__ void column_bits(const HeatmapTcArgs& a, int b, const CropInfo& ci, int lane,
                                            uint32_t (&words)[5]) {
  const uint8_t* mb = crop_mask(a, b);
  bool v[5];
#pragma unroll
  for (int g = 0; g < 5; ++g) {
    const int col = 32 * g + lane;
    v[g] = false;
    if (col < ci.len0 + ci.len1) {
      const bool m1 = col >= ci.off1;
      const int k = (m1 ? ci.kmin1 : ci.kmin0) + (col - (m1 ? ci.off1 : 0));
      v[g] = k < a.K && mb[(m1 ? a.K : 0) + k] != 0;
    }
  }
#pragma unroll
  for (int g = 0; g < 5; ++g) words[g] = __ballot_sync(0xffffffffu, v[g]);
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

// One 128-channel stage held in ring slot ST: eight K=16 steps (two 64-channel
// halves x four) into the accumulator at column dcol. The tensor-memory base is
// 0 (checked after allocation), so every A address and B-descriptor offset is a
// compile-time constant: the issuing thread only adds them to fixed registers.
#ifndef GKD_MMA_X8
#define GKD_MMA_X8 1
#endif
template <int ST>
__device__ __forceinline__ void issue_stage(uint32_t dcol, uint64_t bdesc0, uint32_t idesc, uint32_t first) {
  uint32_t av[8];
  uint64_t bv[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int hs = t >> 2, kk = t & 3;
    av[t] = kColA + ST * 64 + hs * 32 + kk * 8;
    bv[t] = bdesc0 + static_cast<uint64_t>((ST * kBBytes + hs * kBSubBytes + kk * 32) >> 4);
  }
#if GKD_MMA_X8
  umma_ts_f16_x8_elect(dcol, av, bv, idesc, first);   // one elect for the eight
#else
#pragma unroll
  for (int t = 0; t < 8; ++t) umma_ts_f16_elect(dcol, av[t], bv[t], idesc, t == 0 ? first : 1u);
#endif
}

__device__ __forceinline__ void set_abort(Smem* ctl, unsigned* err, unsigned bits) {
  ctl->abort_flag = 1;
  atomicOr(err, bits);
}

// Unit ring, scheduler side: once every other warp has read the slot's
// previous unit (bounded wait, one decision for the warp), fill slot k and
// publish it (the arrive releases the fields to the acquiring waiters).
__device__ __forceinline__ bool unit_publish(Smem* ctl, uint32_t k, int b, int j, int last, const CropInfo& ci,
                                             const uint32_t (&cb)[5], uint64_t lim, volatile int* abortp,
                                             unsigned* err, int lane) {
  const uint32_t slot = k % kUnitSlots;
  const bool okw = k < kUnitSlots || mbar_wait_bounded(&ctl->uempty[slot], ((k / kUnitSlots) & 1) ^ 1, lim, abortp);
  if (!__all_sync(0xffffffffu, okw)) {
    if (lane == 0) set_abort(ctl, err, kErrTimeout);
    return false;
  }
  if (lane == 0) {
    UnitInfo& u = ctl->units[slot];
    u.b = b;
    u.j = j;
    u.last = last;
    u.ci = ci;
#pragma unroll
    for (int g = 0; g < 5; ++g) u.colbits[g] = cb[g];
    mbar_arrive(&ctl->ufull[slot]);
  }
  __syncwarp();
  return true;
}

// Unit ring, reader side: wait until unit k is published (bounded, one decision
// for the warp). The caller reads what it needs from the slot, then releases it.
__device__ __forceinline__ bool unit_wait(Smem* ctl, uint32_t k, uint64_t lim, volatile int* abortp, unsigned* err,
                                          int lane) {
  const bool okw = mbar_wait_bounded(&ctl->ufull[k % kUnitSlots], (k / kUnitSlots) & 1, lim, abortp);
  if (__all_sync(0xffffffffu, okw)) return true;
  if (lane == 0) set_abort(ctl, err, kErrTimeout);
  return false;
}

__device__ __forceinline__ void unit_release(Smem* ctl, uint32_t k, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(&ctl->uempty[k % kUnitSlots]);
}

__device__ __forceinline__ float2 f2sub(float2 b, float2 a) {   // b - a, one rounding
  return __ffma2_rn(a, make_float2(-1.f, -1.f), b);
}

// Pixel layout of a unit (rows Y0..Y0+3, Y0 = 4 vb - 2; columns X0..X0+31):
// TMEM lane 32 q + 16 hf + 8 e + j  <->  pixel (Y0 + 2 hf + e, X0 + 8 q + j).
// All four rows read the same two source rows, so a producer thread owns the
// whole column of four pixels at one X (lanes j, j+8 of both 16-lane halves).
struct Column4 {
  int X;
  int L[4];                   // slab lines of taps (r0,c0) (r0,c1) (r1,c0) (r1,c1), within a half
  float2 lx;                  // x weight
  float2 ly[4];               // y weight of rows Y0 .. Y0+3
};

__device__ __forceinline__ Column4 column_geometry(const HeatmapTcArgs& a, int vb, int ub, int q, int j) {
  Column4 cg;
  const int Y0 = kUnitRows * vb - 2;
  cg.X = kUnitCols * ub + 8 * q + j;
  int r0 = 0, r1 = 0, c0, c1;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    int i0, i1;
    float l;
    src_taps(Y0 + r, a.h, i0, i1, l);
    r0 = i0;          // the same for all four rows (clamped to 0 on the first band)
    r1 = i1;
    cg.ly[r] = make_float2(l, l);
  }
  float lxx;
  src_taps(cg.X, a.w, c0, c1, lxx);
  // slab rows hold source rows vb-1, vb; on the first band r0 = 0 -> slab row 1 and
  // every y weight is 0, so the second tap row only needs to stay inside the slab
  const int sr0 = r0 - (vb - 1);
  const int sr1 = min(r1 - (vb - 1), 1);
  const int sc0 = c0 - (8 * ub - 1), sc1 = c1 - (8 * ub - 1);
  cg.L[0] = sr0 * kSlabCols + sc0;
  cg.L[1] = sr0 * kSlabCols + sc1;
  cg.L[2] = sr1 * kSlabCols + sc0;
  cg.L[3] = sr1 * kSlabCols + sc1;
  cg.lx = make_float2(lxx, lxx);
  return cg;
}

// One channel pair of the four-pixel column: x-lerps on both source rows, then
// four y-lerps; returns the packed bf16x2 words of rows 0..3.
__device__ __forceinline__ void lerp_column(float2 f00, float2 f01, float2 f10, float2 f11, const Column4& cg,
                                            uint32_t (&o)[4]) {
  const float2 t0 = __ffma2_rn(cg.lx, f2sub(f01, f00), f00);
  const float2 t1 = __ffma2_rn(cg.lx, f2sub(f11, f10), f10);
  const float2 dt = f2sub(t1, t0);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float2 u = __ffma2_rn(cg.ly[r], dt, t0);
    o[r] = pack_bf16x2(u.x, u.y);
  }
}

__device__ __forceinline__ float2 bf16lo_hi(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 ld_shared_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// One stage (128 channels) of one producer thread: its column of four pixels x
// 32 channels, written to the A stage at tensor-memory address `acol` (lane
// quadrant base, column of the stage). Channel group r (0..3) of sub-chunk hs
// holds channels 64 hs + 16 r + 4 cq .. +3, i.e. columns 8 r + 2 cq, +1 of the
// sub-chunk: repetition r of the 16x256b.x4 store. fp32 slabs hold 32 channels
// per 128-byte plane line, bf16 slabs 64. tap[k] is the shared address of tap k
// in the stage's first plane (slab stage base + line + swizzled chunk); the
// stage base is 1024-byte aligned, so flipping chunk bits 4-6 of the sum is
// the same as flipping them in the in-slab offset. F5D: the planes are one box
// of 20 lines each (pitch 2560 B, which shifts the swizzle row by 4 from plane
// to plane) instead of separate 3 KB boxes.
template <bool BF16, bool F5D>
__device__ __forceinline__ void produce_stage(const uint32_t (&tap)[4], const Column4& cg, uint32_t acol) {
  constexpr uint32_t plane_bytes = F5D ? kSlabLines * 128u : static_cast<uint32_t>(kPlaneSplit);
  constexpr uint32_t f20 = F5D ? 1u : 0u;
  // kStoreReps repetitions of the 16x256b pattern per store: 4 groups per store
  // (one store per sub-chunk and half quadrant) or 2 (half the live registers)
#pragma unroll
  for (int hr = 0; hr < 8 / kStoreReps; ++hr) {
    const int hs = hr / (4 / kStoreReps);
    uint32_t rows01[4 * kStoreReps], rows23[4 * kStoreReps];
#pragma unroll
    for (int r2 = 0; r2 < kStoreReps; ++r2) {
      const int r = (hr % (4 / kStoreReps)) * kStoreReps + r2;   // channel group within the sub-chunk
      uint32_t o[2][4];   // o[p][row]: channel pair p of the group, pixel row 0..3
      if (!BF16) {
        const int plane = 2 * hs + (r >> 1);
        const uint32_t flip = ((static_cast<uint32_t>(r & 1) ^ (f20 & static_cast<uint32_t>(r >> 1))) << 6);
        const uint32_t po = static_cast<uint32_t>(plane) * plane_bytes;
        const float4 f00 = ld_shared_f4((tap[0] ^ flip) + po);
        const float4 f01 = ld_shared_f4((tap[1] ^ flip) + po);
        const float4 f10 = ld_shared_f4((tap[2] ^ flip) + po);
        const float4 f11 = ld_shared_f4((tap[3] ^ flip) + po);
        lerp_column(make_float2(f00.x, f00.y), make_float2(f01.x, f01.y), make_float2(f10.x, f10.y),
                    make_float2(f11.x, f11.y), cg, o[0]);
        lerp_column(make_float2(f00.z, f00.w), make_float2(f01.z, f01.w), make_float2(f10.z, f10.w),
                    make_float2(f11.z, f11.w), cg, o[1]);
      } else {
        const uint32_t flip = (static_cast<uint32_t>(2 * r) ^ (f20 * 4u * static_cast<uint32_t>(hs & 1))) << 4;
        const uint32_t po = static_cast<uint32_t>(hs) * plane_bytes;
        const uint2 u00 = ld_shared_u2((tap[0] ^ flip) + po);
        const uint2 u01 = ld_shared_u2((tap[1] ^ flip) + po);
        const uint2 u10 = ld_shared_u2((tap[2] ^ flip) + po);
        const uint2 u11 = ld_shared_u2((tap[3] ^ flip) + po);
        lerp_column(bf16lo_hi(u00.x), bf16lo_hi(u01.x), bf16lo_hi(u10.x), bf16lo_hi(u11.x), cg, o[0]);
        lerp_column(bf16lo_hi(u00.y), bf16lo_hi(u01.y), bf16lo_hi(u10.y), bf16lo_hi(u11.y), cg, o[1]);
      }
      // lanes (jx, jx + 8) of a 16-lane half are pixel rows (0, 1) or (2, 3)
      rows01[4 * r2 + 0] = o[0][0];
      rows01[4 * r2 + 1] = o[1][0];
      rows01[4 * r2 + 2] = o[0][1];
      rows01[4 * r2 + 3] = o[1][1];
      rows23[4 * r2 + 0] = o[0][2];
      rows23[4 * r2 + 1] = o[1][2];
      rows23[4 * r2 + 2] = o[0][3];
      rows23[4 * r2 + 3] = o[1][3];
    }
    const uint32_t col = static_cast<uint32_t>(hs * 32 + (hr % (4 / kStoreReps)) * 8 * kStoreReps);
    if (kStoreReps == 4) {
      tmem_st_16x256b_x4(acol + col, reinterpret_cast<const uint32_t(&)[16]>(rows01));
      tmem_st_16x256b_x4(acol + (16u << 16) + col, reinterpret_cast<const uint32_t(&)[16]>(rows23));
    } else if (kStoreReps == 1) {
      tmem_st_16x256b_x1(acol + col, reinterpret_cast<const uint32_t(&)[4]>(rows01));
      tmem_st_16x256b_x1(acol + (16u << 16) + col, reinterpret_cast<const uint32_t(&)[4]>(rows23));
    } else {
      tmem_st_16x256b_x2(acol + col, reinterpret_cast<const uint32_t(&)[8]>(rows01));
      tmem_st_16x256b_x2(acol + (16u << 16) + col, reinterpret_cast<const uint32_t(&)[8]>(rows23));
    }
  }
}

// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) heatmap_tc_kernel(const __grid_constant__ HeatmapTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bring = smem + kSlabStages * kSlabBytes;          // kernel-row stages
  uint8_t* epi_buf = bring + kStages * kBBytes;
  Smem* ctl = reinterpret_cast<Smem*>(epi_buf + 2 * kEpiBufBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
#ifdef GKD_TRACE
  if (tid == 0 && blockIdx.x < 1024) g_entry[blockIdx.x] = global_timer_ns();
#endif

  const int H = 4 * a.h, W = 4 * a.w;
  const int nbands = (H + 2 + kUnitRows - 1) / kUnitRows;
  const int ncb = (W + kUnitCols - 1) / kUnitCols;
  const long long nU = static_cast<long long>(nbands) * ncb;
  const int nchunks = (a.C + kChunk - 1) / kChunk;
  const long long P = static_cast<long long>(H) * W;

  // ---------------- prologue: barriers, TMEM ----------------
  if (tid == 0) {
    for (int s = 0; s < kUnitSlots; ++s) {
      mbar_init(&ctl->ufull[s], 1);                   // the scheduler
      mbar_init(&ctl->uempty[s], kNumWarps - 1);      // every other warp
    }
    mbar_init(&ctl->clc_bar, 1);
    for (int s = 0; s < kSlabStages; ++s) {
      mbar_init(&ctl->sfull[s], 1);
      mbar_init(&ctl->sempty[s], kProdGroupWarps);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->bfull[s], 1);                   // kernel-row TMA arming (+ bytes)
      mbar_init(&ctl->ready[s], kProdGroupWarps);     // the stage's producer group
      mbar_init(&ctl->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctl->accfull[t], 1);
      mbar_init(&ctl->accempty[t], kNumEpiWarps);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpTmaB && lane < 1 + kKernMaps) {
    tma_prefetch_desc(lane == 0 ? &a.tmap_feat : &a.tmap_kern[lane - 1]);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  // B * nU < 2^32 for every size the boundary accepts (65535 crops x 257 x 32 units)
  const uint32_t nU32 = static_cast<uint32_t>(nU);
#ifdef GKD_TRACE
  if (tid == 0 && blockIdx.x < 1024) g_cta[blockIdx.x][0] = global_timer_ns();
#endif
  const uint64_t lim = a.wait_limit_ns;
  volatile int* abortp = &ctl->abort_flag;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == kWarpTma) {
    // ---------------------------------------------------------------- TMA: feature slabs
    uint32_t it = 0, st = 0, ph = 0;
    bool ok = true;
    const uint32_t slab_bytes = (a.feat_bf16 ? 2 : 4) * kPlaneBytes;
    const int nplanes = a.feat_bf16 ? 2 : 4, plane_ch = a.feat_bf16 ? 64 : 32;
    for (uint32_t k = 0; ok; ++k) {
      if (!unit_wait(ctl, k, lim, abortp, a.err, lane)) break;
      const UnitInfo& ui = ctl->units[k % kUnitSlots];
      const int b = ui.b, j = ui.j;
      const bool last = ui.last != 0;
      unit_release(ctl, k, lane);
      if (last) break;
      const int vb = j / ncb, ub = j % ncb;
      for (int ch = 0; ch < nchunks; ++ch, ++it) {
        const bool okw = it < kSlabStages || mbar_wait_bounded(&ctl->sempty[st], ph ^ 1, lim, abortp);
        if (!__all_sync(0xffffffffu, okw)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        if (lane == 0) {
          GKD_TR(0, it);
          uint8_t* sp = smem + st * kSlabBytes;
          uint64_t* fb = &ctl->sfull[st];
          mbar_arrive_expect_tx(fb, slab_bytes);
          const int c0 = ch * kChunk;
          if (a.feat_5d) {
            tma_load_5d(sp, &a.tmap_feat, fb, 0, 8 * ub - 1, vb - 1, c0 / plane_ch, b);
          } else {
            for (int p = 0; p < nplanes; ++p)
              tma_load_4d(sp + p * kPlaneSplit, &a.tmap_feat, fb, c0 + p * plane_ch, 8 * ub - 1, vb - 1, b);
          }
          GKD_TR(1, it);
        }
        __syncwarp();
        if (++st == kSlabStages) { st = 0; ph ^= 1; }
      }
    }
    // drain: no load issued by this warp may still be landing in shared memory
    if (lane == 0) {
      for (uint32_t k = 0; k < kSlabStages && k < it; ++k) {
        const uint32_t last = it - 1 - k;
        if (!mbar_wait_drain(&ctl->sfull[last % kSlabStages], (last / kSlabStages) & 1, lim))
          atomicOr(a.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else if (warp == kWarpTmaB) {
    // ---------------------------------------------------------------- TMA: kernel rows (B operand)
    uint32_t it = 0, st = 0, ph = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      if (!unit_wait(ctl, k, lim, abortp, a.err, lane)) break;
      const UnitInfo& ui = ctl->units[k % kUnitSlots];
      const int b = ui.b;
      const CropInfo ci = ui.ci;
      const bool last = ui.last != 0;
      unit_release(ctl, k, lane);
      if (last) break;
      const int bk = a.kern_shared ? 0 : b;
      const uint32_t bytes = 2 * (ci.len0 + ci.len1) * 128;
      const CUtensorMap* km0 = ci.len0 ? &a.tmap_kern[(ci.len0 >> 3) - 1] : nullptr;
      const CUtensorMap* km1 = ci.len1 ? &a.tmap_kern[(ci.len1 >> 3) - 1] : nullptr;
      for (int ch = 0; ch < nchunks; ++ch, ++it) {
        const bool okw = it < kStages || mbar_wait_bounded(&ctl->empty[st], ph ^ 1, lim, abortp);
        if (!__all_sync(0xffffffffu, okw)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t* bp = bring + st * kBBytes;
          uint64_t* fb = &ctl->bfull[st];
          mbar_arrive_expect_tx(fb, bytes);
          const int c0 = ch * kChunk;
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
            uint8_t* bdst = bp + hs * kBSubBytes;
            if (km0) tma_load_4d(bdst, km0, fb, c0 + hs * kSub, ci.kmin0, 0, bk);
            if (km1) tma_load_4d(bdst + ci.off1 * 128, km1, fb, c0 + hs * kSub, ci.kmin1, 1, bk);
          }
        }
        __syncwarp();
        if (++st == kStages) { st = 0; ph ^= 1; }
      }
    }
    if (lane == 0) {
      for (uint32_t k = 0; k < kStages && k < it; ++k) {
        const uint32_t last = it - 1 - k;
        // bfull[] completes on this warp's own bytes alone, so the drain ends as
        // soon as its copies have landed, aborted run or not
        if (!mbar_wait_drain(&ctl->bfull[last % kStages], (last / kStages) & 1, lim)) atomicOr(a.err, kErrTimeout);
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    // The whole warp runs the role, converged: it waits, computes the crop's
    // size and the descriptors (warp-uniform values, kept in uniform
    // registers), and one elected lane issues each tcgen05.mma and commit. Per
    // stage: two waits, eight MMAs, one commit.
    {
      uint32_t it = 0, v = 0, st = 0, ph = 0;
#ifdef GKD_TRACE
      unsigned long long trace_sum_n = 0;
#endif
      const uint64_t bdesc0 = make_bdesc(smem_u32(bring));
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        if (!unit_wait(ctl, k, lim, abortp, a.err, lane)) {
          ok = false;
          break;
        }
        const UnitInfo& ui = ctl->units[k % kUnitSlots];
        const int n = ui.ci.n;
        const bool last = ui.last != 0;
        unit_release(ctl, k, lane);
        if (last) break;
        const uint32_t idesc = make_idesc(n);
#ifdef GKD_TRACE
        trace_sum_n += n;
#endif
        const int buf = v & 1;
        const uint32_t dcol = buf ? kMaxN : 0u;
        const bool okw = v < 2 || mbar_wait_bounded(&ctl->accempty[buf], ((v >> 1) & 1) ^ 1, lim, abortp);
        if (!__all_sync(0xffffffffu, okw)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        if (lane == 0) GKD_TR(13, v);
        tc_fence_after();
        for (int ch = 0; ch < nchunks; ++ch, ++it) {
          if (lane == 0) GKD_TR(4, it);
          const bool okw2 = mbar_wait_bounded(&ctl->bfull[st], ph, lim, abortp) &&
                            mbar_wait_bounded(&ctl->ready[st], ph, lim, abortp);
          if (!__all_sync(0xffffffffu, okw2)) {
            if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) GKD_TR(2, it);
          const uint32_t first = ch > 0 ? 1u : 0u;
          if (st == 0) {
            issue_stage<0>(dcol, bdesc0, idesc, first);
          } else if (st == 1) {
            issue_stage<1>(dcol, bdesc0, idesc, first);
          } else {
            issue_stage<2>(dcol, bdesc0, idesc, first);
          }
          umma_commit_elect(&ctl->empty[st]);
          if (lane == 0) GKD_TR(3, it);
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit_elect(&ctl->accfull[buf]);
        if (lane == 0) GKD_TR(14, v);
        ++v;
      }
      // drain: every MMA issued by this warp has completed before teardown
      if (it > 0) {
        umma_commit_elect(&ctl->drain);
        const bool drained = mbar_wait_drain(&ctl->drain, 0, lim);
        if (lane == 0 && !drained) atomicOr(a.err, kErrTimeout);
      }
#ifdef GKD_TRACE
      if (lane == 0 && blockIdx.x < 1024) {
        g_cta[blockIdx.x][1] = global_timer_ns();
        g_cta[blockIdx.x][2] = v;
        g_cta[blockIdx.x][3] = trace_sum_n;
      }
#endif
    }
    __syncwarp();
  } else if (warp < kWarpProd0) {
    // ---------------------------------------------------------------- epilogue
    // TMEM -> registers -> padded shared tile [column][row][X] -> float4 rows of the heatmaps
    const int q = warp & 3;
    const int half = (warp - kWarpEpi0) >> 2;       // epilogue set: column groups half, half + kEpiHalves, ...
    const int bar_id = kEpiBarrier + half;
    const int et = tid - (kWarpEpi0 + 4 * half) * 32;   // 0..127 within the set
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const int my_row = 2 * (lane >> 4) + ((lane >> 3) & 1), my_x = 8 * q + (lane & 7);
    // one 10 KB tile per set when there are two sets, two alternating tiles for one set
    const uint32_t epi_base = smem_u32(epi_buf) + (kEpiHalves == 2 ? half * kEpiBufBytes : 0);
    uint32_t v = 0, grp = 0, egrp = 0;
    bool ok = true;
    const bool trace_warp = warp == kWarpEpi0;
    __shared__ uint32_t s_colbits[kNumEpiWarps][5];     // valid-column bits of the current unit's crop, per warp
    uint32_t* colbits = s_colbits[warp - kWarpEpi0];
    for (uint32_t k = 0; ok; ++k) {
      // one decision for the set's four warps (they meet at named barriers below)
      if (!named_bar_and(bar_id, 128,
                         mbar_wait_bounded(&ctl->ufull[k % kUnitSlots], (k / kUnitSlots) & 1, lim, abortp))) {
        if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
        break;
      }
      const UnitInfo& ui = ctl->units[k % kUnitSlots];
      const int b = ui.b, j = ui.j;
      const CropInfo ci = ui.ci;
      const bool last = ui.last != 0;
      if (lane < 5) colbits[lane] = ui.colbits[lane];
      unit_release(ctl, k, lane);                       // its __syncwarp also publishes colbits to the warp
      if (last) break;
      const int buf = v & 1;
      // one decision for the set's four warps: they meet at named barriers below
      const bool okw = named_bar_and(bar_id, 128, mbar_wait_bounded(&ctl->accfull[buf], (v >> 1) & 1, lim, abortp));
      if (!okw) {
        if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0 && trace_warp) GKD_TR(9, v);
      const int Y0 = kUnitRows * (j / ncb) - 2, X0 = kUnitCols * (j % ncb);
      if (a.dec_keys != nullptr) {
        // decode mode: per prompt row, the fp32 mean of the modalities present
        // (their columns are off1 apart), then one peak key per row and tile
        // (warp max, then atomicMax across warps and tiles); no heatmap written
        const int Yp = Y0 + my_row, Xp = X0 + my_x;
        const bool inside = Yp >= 0 && Yp < H && Xp < W;
        const uint32_t pixel = inside ? static_cast<uint32_t>(Yp * W + Xp) : 0u;
        const uint8_t* mb = crop_mask(a, b);
        const bool has0 = ci.len0 > 0, has1 = ci.len1 > 0;
        const int kmin = has0 ? ci.kmin0 : ci.kmin1;
        const int len = has0 ? ci.len0 : ci.len1;
        unsigned long long* keys = a.dec_keys + static_cast<long long>(b) * a.K + kmin;
        bool arrived = false;
        for (int kk = kDecCols * half; kk < len; kk += kDecCols * kEpiHalves) {
          uint32_t v0[kDecCols] = {}, v1[kDecCols] = {};
          if (has0) tmem_ld_32x32b_x8(tmem + lane_off + buf * kMaxN + kk, v0);
          if (has1) tmem_ld_32x32b_x8(tmem + lane_off + buf * kMaxN + ci.off1 + kk, v1);
          tmem_wait_ld();
          if (kk + kDecCols * kEpiHalves >= len) {   // this warp's last load of the accumulator has landed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty[buf]);
            arrived = true;
          }
          // presence of the block's rows: bits 0-7 modality 0, bits 8-15 modality 1
          const int kq = kmin + kk + (lane & 7);
          const bool pres = kq < a.K && ((lane < 8 && has0 && mb[kq] != 0) ||
                                         (lane >= 8 && lane < 16 && has1 && mb[a.K + kq] != 0));
          const uint32_t pbits = __ballot_sync(0xffffffffu, pres);
          unsigned long long mine = 0;   // lane i keeps the key of row kmin + kk + i
#pragma unroll
          for (int i = 0; i < kDecCols; ++i) {
            const bool p0 = (pbits >> i) & 1u;
            const bool p1 = (pbits >> (8 + i)) & 1u;
            if (!p0 && !p1) continue;
            const float f0 = __uint_as_float(v0[i]), f1 = __uint_as_float(v1[i]);
            const float f = (p0 && p1) ? __fmul_rn(__fadd_rn(f0, f1), 0.5f) : (p0 ? f0 : f1);
            uint32_t hi, lo;
            peak_key(f, pixel, inside, hi, lo);
            const unsigned long long key = warp_max_key(hi, lo);
            if (lane == i) mine = key;
          }
          if (mine != 0) atomicMax(keys + kk + lane, mine);
        }
        if (!arrived) {   // this set had no block of the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->accempty[buf]);
        }
        if (lane == 0 && trace_warp) GKD_TR(10, v);
        ++v;
        continue;
      }
      float* hb = a.heat + static_cast<long long>(b) * a.M * a.K * P;
      const int shift0 = ci.kmin0, shift1 = a.K + ci.kmin1 - ci.off1;

      const int ngroups = ci.n / kEpiCols;
      if (half >= ngroups) {   // no column group for this set: release the accumulator now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->accempty[buf]);
        ++v;
        continue;
      }
      // software-pipelined: the TMEM load of the set's next group (and its
      // validity bits) are in flight while the current group goes through
      // shared memory to HBM
      uint32_t cur[16], nxt[16];
      tmem_ld_32x32b_x16(tmem + lane_off + buf * kMaxN + half * kEpiCols, cur);
      auto group_bits = [&](int n0) { return (colbits[n0 >> 5] >> (n0 & 31)) & 0xFFFFu; };
      uint32_t bits = group_bits(half * kEpiCols);
      tmem_wait_ld_regs(cur);
      for (int gi = half; gi < ngroups; gi += kEpiHalves) {
        const int n0 = gi * kEpiCols;
        const bool more = gi + kEpiHalves < ngroups;
        uint32_t bits_next = 0;
        if (more) {
          tmem_ld_32x32b_x16(tmem + lane_off + buf * kMaxN + n0 + kEpiHalves * kEpiCols, nxt);
          bits_next = group_bits(n0 + kEpiHalves * kEpiCols);
        } else {   // every load of this accumulator by this warp has landed: let the MMA reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->accempty[buf]);
        }
        if (lane == 0 && trace_warp) GKD_TR(11, egrp);
        if (bits != 0) {   // uniform across the set's four warps (same crop)
          const uint32_t sb = epi_base + (kEpiHalves == 1 ? (grp & 1) * kEpiBufBytes : 0);
          // one tile per set: wait until every warp of the set has read the previous group
          if (kEpiHalves == 2 && grp > 0) named_bar_sync(bar_id, 128);
          // stage this thread's pixel: [col][row][X], row stride kEpiStride floats
#pragma unroll
          for (int c = 0; c < kEpiCols; ++c)
            st_shared_f32(sb + ((c * kUnitRows + my_row) * kEpiStride + my_x) * 4, cur[c]);
          named_bar_sync(bar_id, 128);
          if (lane == 0 && trace_warp) GKD_TR(12, egrp);
          // each thread writes 4 float4 (4 consecutive X of one column and row)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int f = i * 128 + et;
            const int c = f >> 5, r = (f >> 3) & 3, x4 = f & 7;
            if ((bits >> c) & 1u) {
              const int Y = Y0 + r, X = X0 + 4 * x4;
              if (Y >= 0 && Y < H && X < W) {
                const float4 val = ld_shared_f4(sb + ((c * kUnitRows + r) * kEpiStride + 4 * x4) * 4);
                const int n = n0 + c;
                const int row = n + (n < ci.off1 ? shift0 : shift1);
                __stcs(reinterpret_cast<float4*>(hb + static_cast<long long>(row) * P +
                                                 static_cast<long long>(Y) * W + X),
                       val);
              }
            }
          }
          ++grp;   // staging buffers alternate only between groups that passed the barrier
        }
        if (lane == 0 && trace_warp) GKD_TR(15, egrp);
        ++egrp;
        if (more) {
          tmem_wait_ld_regs(nxt);
#pragma unroll
          for (int c = 0; c < kEpiCols; ++c) cur[c] = nxt[c];
          bits = bits_next;
        }
      }
      if (lane == 0 && trace_warp) GKD_TR(10, v);
      ++v;
    }
  } else if (warp == kWarpSched) {
    // ---------------------------------------------------------------- unit scheduler
    // Work comes from the hardware's CTA queue: first this CTA's own unit (its
    // blockIdx), then, one at a time, the units of CTAs of the grid that have not
    // started yet, taken over by cluster launch control (a cancelled CTA never
    // runs). Units of crops without a valid row are dropped here; every other
    // unit goes into the ring with its crop's row segments and column bits, so
    // that no other role reads the mask. The last entry is a stop marker.
    const bool dec = a.dec_keys != nullptr;
    const bool same_rows = a.kern_shared && a.mask_batch_stride == 0;   // every crop has the same rows
    uint32_t k = 0, cph = 0, item = blockIdx.x;
    bool ok = true, pending = false, have = true;
    if (tmem != 0) {
      // the MMA issue path assumes the whole tensor memory from column 0 (the only
      // place a 512-column allocation can land); anything else: no work
      if (lane == 0) atomicOr(a.err, kErrBounds);
      have = false;
    }
    auto request = [&]() {       // one cancellation request in flight at a time
      if (lane == 0) {
        fence_proxy_async_smem();                       // the last response was read before it is rewritten
        mbar_arrive_expect_tx(&ctl->clc_bar, 16);
        clc_try_cancel(&ctl->clc_resp, &ctl->clc_bar);
      }
      __syncwarp();
      pending = true;
    };
    // 1: a CTA was cancelled (its unit is now `item`), 0: the queue is empty, -1: the wait failed
    auto response = [&](bool drain) -> int {
      const bool got = drain ? mbar_wait_drain(&ctl->clc_bar, cph, lim)
                             : mbar_wait_bounded(&ctl->clc_bar, cph, lim, abortp);
      if (!__all_sync(0xffffffffu, got)) return -1;
      pending = false;
      cph ^= 1;
      uint32_t x;
      if (!clc_query(&ctl->clc_resp, x)) return 0;
      item = x;
      return 1;
    };
    if (have) request();
    int cur = -1;
    CropInfo ci{};
    uint32_t cb[5] = {0u, 0u, 0u, 0u, 0u};
    while (have) {
      const int b = static_cast<int>(item / nU32), j = static_cast<int>(item % nU32);
      if ((same_rows ? 0 : b) != cur) {
        ci = crop_info(a, b, lane, dec);
        if (!dec) column_bits(a, b, ci, lane, cb);
        cur = same_rows ? 0 : b;
      }
      if (ci.n > 0) {
        if (!unit_publish(ctl, k, b, j, 0, ci, cb, lim, abortp, a.err, lane)) {
          ok = false;
          break;
        }
        ++k;
      }
      have = false;
      if (pending) {
        const int r = response(false);
        if (r < 0) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        if (r > 0) {
          have = true;
          request();
        }
      }
    }
    if (ok) ok = unit_publish(ctl, k, 0, 0, 1, ci, cb, lim, abortp, a.err, lane);
    // A response still in flight must land before the CTA exits. After a failure
    // the queued CTAs are taken over without doing their units, so that none of
    // them starts only to wait out the limit again.
    while (pending) {
      const int r = response(true);
      if (r < 0 && lane == 0) atomicOr(a.err, kErrTimeout);
      if (r <= 0) break;
      request();
    }
  } else {
    // ---------------------------------------------------------------- upsample producers
    const int q = warp & 3;                             // lane quadrant this warp may write
    const int grp = (warp - kWarpProd0) / kProdGroupWarps;
    const int jx = lane >> 2, cq = lane & 3;            // column within the quadrant, 4-channel group
    const bool skip_first = (a.debug_flags & kDbgSkipProducerArrive) != 0;
    uint32_t it = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      if (!unit_wait(ctl, k, lim, abortp, a.err, lane)) break;
      const int j = ctl->units[k % kUnitSlots].j;
      const bool last = ctl->units[k % kUnitSlots].last != 0;
      unit_release(ctl, k, lane);
      if (last) break;
      // this group's first stage of the unit, if it has one
      int ch = (grp - static_cast<int>(it % kProdGroups) + kProdGroups) % kProdGroups;
      if (ch >= nchunks) { it += nchunks; continue; }
      const Column4 cg = column_geometry(a, j / ncb, j % ncb, q, jx);
      // per tap: the tap's line inside a plane plus the swizzled 16-byte chunk of
      // this thread's first channel group; the other groups flip chunk bits
      uint32_t base[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t L = static_cast<uint32_t>(cg.L[k]);
        base[k] = a.feat_bf16
                      ? (L * 128u | (((static_cast<uint32_t>(cq) >> 1) ^ (L & 7u)) << 4)) + ((cq & 1u) << 3)
                      : (L * 128u | ((static_cast<uint32_t>(cq) ^ (L & 7u)) << 4));
      }
      for (; ch < nchunks; ch += kProdGroups) {
        const uint32_t s_it = it + ch;
        const uint32_t st = s_it % kStages, ph = (s_it / kStages) & 1;
        const uint32_t ss = s_it % kSlabStages, sph = (s_it / kSlabStages) & 1;
        bool okw = mbar_wait_bounded(&ctl->sfull[ss], sph, lim, abortp);
        if (okw && s_it >= kStages) okw = mbar_wait_bounded(&ctl->empty[st], ph ^ 1, lim, abortp);
        if (!__all_sync(0xffffffffu, okw)) {
          if (lane == 0) set_abort(ctl, a.err, kErrTimeout);
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0 && (warp - kWarpProd0) % kProdGroupWarps == 0) GKD_TR(6, s_it);
        const uint32_t sp = smem_base + ss * kSlabBytes;   // 1024-byte aligned
        const uint32_t acol = tmem + kColA + st * 64 + (static_cast<uint32_t>(32 * q) << 16);
        uint32_t tap[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          tap[k] = sp + base[k];
          // opaque per stage: keeps the compiler from hoisting the 16 swizzled tap
          // addresses of the stage out of the loop (registers it does not have)
          asm volatile("" : "+r"(tap[k]));
        }
        if (a.feat_bf16) {
          if (a.feat_5d) produce_stage<true, true>(tap, cg, acol);
          else produce_stage<true, false>(tap, cg, acol);
        } else {
          if (a.feat_5d) produce_stage<false, true>(tap, cg, acol);
          else produce_stage<false, false>(tap, cg, acol);
        }
        if (lane == 0 && (warp - kWarpProd0) % kProdGroupWarps == 0) GKD_TR(7, s_it);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ctl->sempty[ss]);                 // slab consumed (loads completed above)
          if (!(skip_first && s_it == 0)) mbar_arrive(&ctl->ready[st]);
        }
        if (lane == 0 && (warp - kWarpProd0) % kProdGroupWarps == 0) GKD_TR(8, s_it);
      }
      it += nchunks;
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

#ifdef GKD_TRACE
extern "C" __attribute__((visibility("default"))) int gkd_trace_cta(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, tc::g_cta, sizeof(tc::g_cta)));
}
extern "C" __attribute__((visibility("default"))) int gkd_trace_entry(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, tc::g_entry, sizeof(tc::g_entry)));
}
extern "C" __attribute__((visibility("default"))) int gkd_trace_read(void* host, int clear) {
  cudaError_t e = cudaMemcpyFromSymbol(host, tc::g_trace, sizeof(tc::g_trace));
  if (e == cudaSuccess && clear) {
    static unsigned long long zero[16][2048];
    e = cudaMemcpyToSymbol(tc::g_trace, zero, sizeof(zero));
  }
  return static_cast<int>(e);
}
#endif

static bool encode(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                   const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
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
  a.feat_5d = 0;
  const cuuint64_t elt = a.feat_bf16 ? 2 : 4;
  const cuuint64_t plane_ch = a.feat_bf16 ? 64 : 32;       // channels of one 128-byte slab plane
  const CUtensorMapDataType fdt = a.feat_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (a.C % plane_ch == 0) {
    // channels split as (plane, C / plane) so one box brings every plane of a 128-channel stage
    const cuuint64_t dims[5] = {plane_ch, w, h, C / plane_ch, B};
    const cuuint64_t strides[4] = {C * elt, w * C * elt, 128, h * w * C * elt};
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(plane_ch), tc::kSlabCols, tc::kSlabRows,
                               static_cast<cuuint32_t>(tc::kChunk / plane_ch), 1};
    if (!encode(enc, &a.tmap_feat, fdt, 5, feat, dims, strides, box)) {
      *why = "tensor map encoding failed for the feature map";
      return cudaErrorInvalidValue;
    }
    a.feat_5d = 1;
  } else {
    const cuuint64_t dims[4] = {C, w, h, B};
    const cuuint64_t strides[3] = {C * elt, w * C * elt, h * w * C * elt};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(plane_ch), tc::kSlabCols, tc::kSlabRows, 1};
    if (!encode(enc, &a.tmap_feat, fdt, 4, feat, dims, strides, box)) {
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
      if (!encode(enc, &a.tmap_kern[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, kern, dims, strides, box)) {
        *why = "tensor map encoding failed for the kernel rows";
        return cudaErrorInvalidValue;
      }
    }
  }
  cudaError_t e = cudaFuncSetAttribute(tc::heatmap_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(tc::kSmemBytes));
  if (e != cudaSuccess) return e;
  const int H = 4 * a.h, W = 4 * a.w;
  const long long nU = static_cast<long long>((H + 2 + tc::kUnitRows - 1) / tc::kUnitRows) *
                       ((W + tc::kUnitCols - 1) / tc::kUnitCols);
  // one CTA per unit: the SMs run one CTA each and take the queued CTAs' units
  // over (cluster launch control), so the grid is the work list
  (void)num_sms;
  const long long units = nU * a.B;
  tc::heatmap_tc_kernel<<<static_cast<unsigned>(units), tc::kThreads, tc::kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gkd
