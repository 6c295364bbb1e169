// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
// Every launcher assumes its arguments were validated by the caller and only
// enqueues work on `stream`; it returns the CUDA launch status.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace gkd {

// Device error word bits (written by kernels, read by gkd_check_device_error).
enum : unsigned {
  kErrTimeout = 1u << 0,   // a bounded wait ran out
  kErrBounds = 1u << 1,    // a bounds or placement check fired (the kernel did no work)
};

// Test hooks for the forced-timeout path (host-set, consumed by the next launch).
enum : unsigned {
  kDbgSkipProducerArrive = 1u << 0,   // upsample producers never signal their first stage
};

cudaError_t launch_norm(const float* rows, const uint8_t* mask, long long nrows, int C, float eps,
                        bool out_bf16, void* out, cudaStream_t stream);

cudaError_t launch_norm_fuse(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C, float eps,
                             bool out_bf16, void* out, uint8_t* out_mask, cudaStream_t stream);

// Image preprocessing of B boxes of one image and the ROI -> image coordinate map (preprocess.cu).
cudaError_t launch_preprocess(const uint8_t* img, int H, int W, const float* boxes, int B, int canvas, float* out,
                              cudaStream_t stream);
cudaError_t launch_roi_to_image(const float* xy, const float* boxes, int B, int K, int canvas, float* out,
                                cudaStream_t stream);

cudaError_t launch_fuse_decode(const float* heat, const uint8_t* mask, long long mask_batch_stride,
                               int B, int M, int K, int H, int W, float* fused, float* xy, float* score,
                               int32_t* idx, uint8_t* valid, cudaStream_t stream);

// keys non-null: decode mode (no heatmap; one peak key per (crop, row) merged into keys)
cudaError_t launch_heatmap_f32(const float* feat, int B, int h, int w, int C, const float* kern,
                               long long kern_batch_stride, const uint8_t* mask, long long mask_batch_stride,
                               int M, int K, float* heat, unsigned long long* keys, int num_sms,
                               cudaStream_t stream);

// Turns peak keys [B][K] into idx / xy / score / valid (decode fused into the heatmap kernels).
cudaError_t launch_finalize_keys(const unsigned long long* keys, const uint8_t* mask, long long mask_batch_stride,
                                 int B, int M, int K, int H, int W, float* xy, float* score, int32_t* idx,
                                 uint8_t* valid, cudaStream_t stream);

constexpr int kKernMaps = 16;   // kernel-row boxes of 8, 16, ..., 128 rows

struct HeatmapTcArgs {
  CUtensorMap tmap_feat;                 // feature slabs: fp32 {32, w, h, C/32, B} or {C, w, h, B}
  CUtensorMap tmap_kern[kKernMaps];      // kernel rows {C, K, M, Bk}, box {64, 8 (i + 1), 1, 1}
  const uint8_t* mask;
  long long mask_batch_stride;
  float* heat;                           // heatmaps (heatmap mode), unused in decode mode
  unsigned long long* dec_keys;          // decode mode: per (crop, row) peak key, zeroed before launch; else null
  int B, h, w, C, M, K;
  int feat_bf16;
  int feat_5d;               // fp32 slab as one 5-D box (C % 32 == 0), else two 4-D boxes
  int kern_shared;           // kernels shared by all crops (batch stride 0)
  unsigned* err;             // device error word
  unsigned long long wait_limit_ns;
  unsigned debug_flags;
};

// Encodes the tensor maps and launches the persistent tcgen05 kernel.
cudaError_t launch_heatmap_tc(HeatmapTcArgs& a, const void* feat, const void* kern,
                              long long kern_batch_stride, int num_sms, cudaStream_t stream,
                              const char** why);

// Contract-then-upsample variant (contract_tc.cu).
struct ContractArgs {
  CUtensorMap tmap_feat;                 // features as [B*h*w][C], box {32 (fp32) or 64 (bf16), 128}
  CUtensorMap tmap_kern[kKernMaps];      // kernel rows, as for HeatmapTcArgs
  const uint8_t* mask;
  long long mask_batch_stride;
  float* G;                              // [B][M][K][h*w] fp32 contraction on the source grid (scratch)
  int B, h, w, C, M, K;
  int feat_bf16;
  int kern_shared;
  unsigned* err;
  unsigned long long wait_limit_ns;
};

cudaError_t launch_contract_first(ContractArgs& a, const void* feat, const void* kern, long long kern_batch_stride,
                                  float* heat, cudaStream_t stream, const char** why);

// Gaussian prototype pooling on the tensor cores (pool_tc.cu).
struct PoolTcArgs {
  CUtensorMap tmap;                      // support features as {C, h*w, B} fp32, box {32, 32, 1}
  const float* kpts;                     // [B][K][2]
  const uint8_t* kmask;                  // [B][K]
  float* proto;
  long long proto_bs;
  int h, w, C, K;
  int N;                                 // channels per CTA (32..256, a multiple of 32)
  float sigma, stride;
  unsigned* err;
  unsigned long long wait_limit_ns;
};

cudaError_t launch_pool_tc(const float* support, int B, int h, int w, int C, const float* kpts,
                           const uint8_t* kmask, int K, float sigma, float stride, float* proto,
                           long long proto_batch_stride, unsigned* err, unsigned long long wait_limit_ns,
                           int num_sms, cudaStream_t stream, const char** why);

// cuTensorMapEncodeTiled resolved through the runtime's driver entry point.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace gkd
