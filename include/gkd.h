/*
 * gkd.h - C ABI of libgkd, a B200 (sm_100a) implementation of the
 * parameter-free detection head of GKDT (General Keypoint Detection
 * Transformer): prompts become 1x1 convolution kernels that are matched against
 * dense query features to give keypoint heatmaps, which are decoded to
 * coordinates.
 *
 * Sources for the operations (titles and sections of the pages that define them):
 *   [CARD]  Asher-1/GKD_GGUF model card, section Model. Architecture bullet:
 *           the detection head has no parameters; it upsamples the features
 *           4x bilinearly, L2-normalises the prompt kernels, applies them as
 *           1x1 convolutions and fuses rows under a mask, with prompts padded
 *           to 80 rows. Prompts bullet: visual prompts are pooled with a
 *           Gaussian of sigma 14; text and visual prompts can be combined row
 *           by row. Output bullet: the peak of each prompt's heatmap on a 96x96
 *           grid, mapped into the ROI's -1..1 space, with a confidence score.
 *   [SUMM]  GKDT: General Keypoint Detection Transformer, summary page,
 *           pipeline paragraph: visual prototypes come from Gaussian weights
 *           on the support image; the prompt kernels are convolved over the
 *           query image's features.
 *   [NOTES] GKDT reading notes (arxiv-cs-cv-2607-00752), section Method:
 *           support features are aggregated into visual keypoint prototypes;
 *           the matching is a normalised convolution.
 *
 * Conventions shared by every entry point:
 *   - Tensor arguments are DEVICE pointers owned by the caller. The library
 *     never frees them, never keeps them after the call returns, allocates no
 *     device memory, and never synchronises the stream (except
 *     gkd_check_device_error). Work is enqueued asynchronously on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream) on the device
 *     that owns the first tensor argument. That device becomes the calling
 *     thread's current device and stays current after the call returns, so
 *     that a following gkd_check_device_error() on the same thread reads the
 *     error word of the device that ran the work.
 *   - Layouts are dense row-major with the last index contiguous, unless a
 *     batch-stride argument says otherwise. Strides are in ELEMENTS.
 *   - Masks are uint8 with 0 (absent) or 1 (present) per entry.
 *   - Arguments are validated on the host before anything is launched. On any
 *     violation the call returns a non-zero gkd_status, launches nothing, and
 *     gkd_last_error() describes the problem. Checks: non-null device pointers,
 *     positive sizes, dtype support, C % 8 == 0, 16-byte alignment of every
 *     tensor base pointer and of every batch stride in bytes, size limits
 *     stated per call.
 *   - Outputs are fully written (entries of invalid rows get the documented
 *     fill value) except where a call says a region is left unspecified.
 *   - Results of kernels with bounded internal waits: if a wait times out the
 *     kernel records it in a device error word and returns early (outputs are
 *     then unspecified); gkd_check_device_error() reports it as
 *     GKD_ERR_TIMEOUT.
 *   - Host threads: every entry point may be called from several threads at
 *     once. gkd_last_error() is per thread. The wait limit
 *     (gkd_set_wait_timeout_ms) and the debug flags (gkd_debug_set_flags) are
 *     process-wide: the flags are consumed by whichever bf16 gkd_heatmap
 *     launch comes next, from any thread.
 */
#ifndef GKD_H_
#define GKD_H_

#include <stdint.h>

#if defined(__GNUC__)
#define GKD_API __attribute__((visibility("default")))
#else
#define GKD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gkd_status {
  GKD_OK = 0,
  GKD_ERR_ARG = 1,      /* null / non-device pointer, bad enum, bad flag */
  GKD_ERR_SHAPE = 2,    /* a size is zero, negative, or beyond a stated limit */
  GKD_ERR_DTYPE = 3,    /* unsupported dtype or dtype combination */
  GKD_ERR_ALIGN = 4,    /* a pointer or byte stride is not 16-byte aligned */
  GKD_ERR_CUDA = 5,     /* a CUDA runtime call failed (launch, attribute, ...) */
  GKD_ERR_TIMEOUT = 6   /* a kernel's bounded wait ran out (see gkd_check_device_error) */
} gkd_status;

typedef enum gkd_dtype {
  GKD_F32 = 0,          /* IEEE binary32 */
  GKD_BF16 = 1          /* bfloat16 (upper half of binary32), stored as 16-bit words */
} gkd_dtype;

/*
 * Step 1: Gaussian prototype pooling of support features ([CARD] Prompts
 * bullet, Gaussian pooling with sigma 14; [SUMM] pipeline paragraph; [NOTES]
 * Method, support features aggregated into visual prototypes).
 *
 *   proto[b,k,:] = sum_ij w_ij * support[b,i,j,:] / sum_ij w_ij,
 *   w_ij = exp(-((X_j - x)^2 + (Y_i - y)^2) / (2 sigma^2)),
 *   X_j = stride_px * (j + 0.5), Y_i = stride_px * (i + 0.5),
 * for keypoints with kmask[b,k] != 0; rows of absent keypoints are set to 0.
 * The weights are evaluated over the whole h x w grid (no truncation).
 *
 *   support  [B][h][w][C] (sdt = GKD_F32 only; GKD_BF16 returns GKD_ERR_DTYPE)
 *   kpts     [B][K][2] fp32, (x, y) in ROI pixels of the support image
 *   kmask    [B][K] uint8
 *   proto    fp32; crop b's rows start at proto + b * proto_batch_stride and are
 *            [K][C] contiguous (proto_batch_stride >= K * C; pass 2*K*C to
 *            write straight into modality 0 of a [B][2][K][C] row tensor).
 * Limits: 1 <= K <= 128, 1 <= h, w <= 256, B <= 65535, sigma_px > 0, stride_px > 0.
 * Computed as one tensor-core GEMM per crop (keypoints x pixels x channels):
 * the weights and features are each carried as a pair of TF32 numbers
 * (x = hi + lo), three products per term, fp32 accumulation in a fixed order
 * (the result does not depend on scheduling); each term is within about
 * 2^-21 of its fp32 product. Features must be finite.
 */
GKD_API gkd_status gkd_pool_prototypes(const void* support, gkd_dtype sdt, int B, int h, int w, int C,
                               const float* kpts, const uint8_t* kmask, int K, float sigma_px,
                               float stride_px, float* proto, long long proto_batch_stride,
                               void* stream);

/*
 * Step 2: L2 normalisation of prompt rows ([CARD] Architecture bullet, kernel
 * rows normalised, prompts padded to 80 rows; [NOTES] Method, normalised
 * convolution).
 *
 *   out[r,:] = rows[r,:] / max(||rows[r,:]||_2, eps)  where mask[r] != 0,
 *   out[r,:] = 0                                       where mask[r] == 0,
 * over the Bk*M*K rows of rows [Bk][M][K][C] (fp32) with mask [Bk][M][K].
 * Sum of squares in fp32, IEEE square root and division. out_dt = GKD_BF16
 * rounds the fp32 quotient to bf16 (nearest, ties to even).
 *   out  [Bk][M][K][C], fp32 or bf16 per out_dt.
 * Limits: 1 <= M <= 2, 1 <= K <= 128, eps > 0, Bk*M*K < 2^31.
 */
GKD_API gkd_status gkd_norm_kernels(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C, float eps,
                            gkd_dtype out_dt, void* out, void* stream);

/*
 * Step 2 with the modality fusion of step 5 moved in front of the contraction
 * ("fusion by linearity"): the heatmap is linear in the kernel row, so the mean
 * of a prompt row's two modality heatmaps ([CARD] Architecture bullet, masked
 * fusion per row; Prompts bullet, text and visual combined row by row) equals
 * the heatmap of the mean of its two normalised rows, and the contraction then
 * runs once per prompt row instead of once per (modality, row).
 *
 *   khat_m   = rows[b,m,k,:] / max(||rows[b,m,k,:]||_2, eps)   (as gkd_norm_kernels)
 *   out[b,k] = (khat_0 + khat_1) * 0.5 in fp32 when both modalities are present,
 *              khat_m when only m is, 0 when none; rounded once to out_dt
 *   out_mask[b,k] = 1 if any modality is present, else 0.
 *   rows [Bk][M][K][C] fp32, mask [Bk][M][K], out [Bk][K][C] (fp32 or bf16),
 *   out_mask [Bk][K] uint8. Pass out and out_mask to gkd_heatmap or
 *   gkd_heatmap_decode with M = 1 (and to gkd_fuse_decode with M = 1).
 * The result differs from the graded fused heatmap only by rounding (a
 * separately checked variant, not the graded path).
 * Limits: 1 <= M <= 2, 1 <= K <= 128, eps > 0, Bk*M*K < 2^31.
 */
GKD_API gkd_status gkd_norm_fuse_kernels(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C,
                                         float eps, gkd_dtype out_dt, void* out, uint8_t* out_mask, void* stream);

/*
 * Steps 3 + 4: bilinear 4x upsample of the query features (align_corners =
 * False, half-pixel source coordinate s = max((d + 0.5)/4 - 0.5, 0), upper
 * neighbour clamped to the last row/column) fused into the 1x1 dynamic-kernel
 * contraction ([CARD] Architecture bullet, 4x bilinear upsample and 1x1
 * prompt kernels; [CARD] Output bullet, 96x96 grid; [SUMM] pipeline paragraph,
 * prompt kernels convolved over the query features):
 *
 *   heat[b,m,k,Y,X] = sum_c kern[b,m,k,c] * U[b,Y,X,c]   for mask[b,m,k] != 0.
 *
 *   feat    [B][h][w][C], fdt = GKD_F32 or GKD_BF16
 *   kern    crop b's rows at kern + b * kern_batch_stride, [M][K][C];
 *           kern_batch_stride = 0 shares one prompt set across all crops.
 *           kdt = GKD_BF16: tensor-core path. U is formed in fp32 and rounded
 *             to bf16 (nearest even); products are summed in fp32.
 *           kdt = GKD_F32 (requires fdt = GKD_F32): fp32 path, U and the sum in
 *             fp32.
 *   mask    crop b's [M][K] at mask + b * mask_batch_stride (0 = shared)
 *   heat    [B][M][K][4h][4w] fp32. Rows with mask == 0 are NOT written
 *           (left unspecified).
 * Limits: up == 4, 1 <= M <= 2, 1 <= K <= 128, M * ceil8(K) <= 160 on the bf16
 *         path, 1 <= h, w <= 256, B <= 65535, C % 8 == 0.
 */
GKD_API gkd_status gkd_heatmap(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                       const void* kern, gkd_dtype kdt, long long kern_batch_stride,
                       const uint8_t* mask, long long mask_batch_stride, int M, int K,
                       float* heat, void* stream);

/*
 * Steps 3 + 4 in the other order ("contract then upsample", a variant beside
 * the graded path): the 1x1 contraction and the 4x bilinear upsample ([CARD]
 * Architecture bullet) are both linear, so
 *
 *   G[b,m,k,i,j]   = sum_c kern[b,m,k,c] * bf16(feat[b,i,j,c])   on the h x w grid,
 *   heat[b,m,k]    = Up(G[b,m,k])   (the rule of gkd_heatmap, applied to G),
 *
 * equals gkd_heatmap's result in exact arithmetic with 16x fewer multiply-adds.
 * Rounding points differ: the features are rounded to bf16 (the tensor-core
 * operand), U is never formed, G is fp32 (tensor-core accumulation) and the
 * upsample of G is fp32; so this is checked against its own definition, not
 * bit for bit against gkd_heatmap. Bound by the heatmap writes (HBM).
 *
 * Arguments as in gkd_heatmap with bf16 kernel rows (no kdt), plus
 *   scratch  [B][M][K][h*w] fp32 device memory owned by the caller (G; rows with
 *            mask 0 are not written), 4-byte aligned.
 * Two launches on `stream` (the contraction, then the upsample).
 * Limits: those of gkd_heatmap's bf16 path.
 */
GKD_API gkd_status gkd_heatmap_contract_first(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                                              const void* kern, long long kern_batch_stride, const uint8_t* mask,
                                              long long mask_batch_stride, int M, int K, float* scratch,
                                              float* heat, void* stream);

/*
 * Steps 3 + 4 + 5 in one pass, heatmaps never written: the contraction of
 * gkd_heatmap, with the per-row masked fusion and peak decode of
 * gkd_fuse_decode done on the accumulators inside the heatmap kernel's
 * epilogue ([CARD] Architecture bullet, masked fusion per prompt row; Output
 * bullet, per-prompt peak mapped to ROI -1..1 with a confidence score).
 *
 * Arguments as in gkd_heatmap (no heat) and gkd_fuse_decode (no fused map);
 * the outputs idx, xy, score and valid equal gkd_fuse_decode's on the
 * heatmaps gkd_heatmap writes, bit for bit: the same fp32 fusion of the same
 * accumulator values and the same first-maximum rule.
 *   scratch  [B][K] uint64 device memory owned by the caller (8-byte aligned),
 *            used as one peak key per (crop, row) merged across pixel tiles;
 *            the call clears it first (asynchronously on `stream`) and leaves
 *            its contents unspecified. Calls that share a scratch buffer must
 *            not overlap on the GPU.
 * Three launches on `stream`: the scratch clear, the heatmap kernel in
 * decode mode, and a small kernel that turns the keys into the outputs.
 * NaN values never win; a valid row whose every fused value is NaN decodes to
 * idx 0 with a NaN score (gkd_fuse_decode does the same).
 * Limits: those of gkd_heatmap.
 */
GKD_API gkd_status gkd_heatmap_decode(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                                      const void* kern, gkd_dtype kdt, long long kern_batch_stride,
                                      const uint8_t* mask, long long mask_batch_stride, int M, int K,
                                      unsigned long long* scratch, float* xy, float* score, int32_t* idx,
                                      uint8_t* valid, void* stream);

/*
 * gkd_heatmap_decode for callers that cannot give the library any device
 * memory: everything it needs beyond its inputs and outputs lives in one
 * statically sized buffer inside the library. This is for code that is
 * handed only its input and output tensors and has no way to allocate (for
 * example a plug-in or inference-server hook without a workspace, or a
 * process that has fixed its device memory budget at start-up and may not
 * call cudaMalloc afterwards). The paper has no counterpart: it is an
 * interface variant of the fused decode, not a step of the method.
 *
 * Arguments and outputs are those of gkd_heatmap_decode without `scratch`;
 * the outputs are the same, bit for bit.
 *   - The peak keys live in a file-scope __device__ array of 131072 entries
 *     (1 MiB), which every GPU that loads the library holds until the process
 *     exits. Calls with B * K > 131072 return GKD_ERR_SHAPE and launch nothing
 *     (use gkd_heatmap_decode with your own scratch for those).
 *   - The first call on a device looks up that array's device address (a
 *     symbol lookup, no allocation) with the device current; make that first
 *     call before any stream capture.
 *   - Each call clears the part of the array it uses, asynchronously on
 *     `stream`, before the heatmap kernel. All calls on a device share the
 *     array and it keeps the last call's contents: calls that overlap on the
 *     GPU (different streams, or different host threads) race on it and give
 *     wrong results. Serialise them.
 *   - The call allocates and frees nothing (no cudaMalloc, cudaFree or
 *     allocating library routine).
 * Limits: those of gkd_heatmap, and B * K <= 131072.
 */
GKD_API gkd_status gkd_heatmap_decode_noalloc(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                                              const void* kern, gkd_dtype kdt, long long kern_batch_stride,
                                              const uint8_t* mask, long long mask_batch_stride, int M, int K,
                                              float* xy, float* score, int32_t* idx, uint8_t* valid, void* stream);

/*
 * Step 5: per-row masked fusion across modalities and peak decode ([CARD]
 * Architecture bullet, masked fusion per prompt row; Prompts bullet, text and
 * visual combined row by row; Output bullet, peak mapped to ROI -1..1 plus a
 * confidence score).
 *
 * For each (b, k): cnt = number of modalities m with mask[b,m,k] != 0;
 *   fused = heat[b,m,k] for the one present modality, or
 *           (heat[b,0,k] + heat[b,1,k]) * 0.5 in fp32 when both are;
 *   idx   = first (lowest row-major index Y*W + X) maximal pixel of fused;
 *   score = fused[idx];
 *   xy    = ((2 X + 1 - W) / W, (2 Y + 1 - H) / H), one IEEE fp32 division each
 *           (= 2 (X + 0.5)/W - 1, correctly rounded);
 *   valid = 1.
 * Rows with cnt == 0: idx = -1, xy = (0, 0), score = 0, valid = 0, fused row 0.
 * Inputs are expected finite. NaN values never win; a valid row whose every
 * fused value is NaN decodes to idx 0, valid 1 and the (NaN) fused value there.
 *
 *   heat   [B][M][K][H][W] fp32 (rows with mask 0 are not read)
 *   mask   crop b's [M][K] at mask + b * mask_batch_stride (0 = shared)
 *   fused  optional [B][K][H][W] fp32 (NULL: not written)
 *   xy [B][K][2] fp32, score [B][K] fp32, idx [B][K] int32, valid [B][K] uint8
 * Limits: 1 <= M <= 2, 1 <= K <= 65535, H * W % 4 == 0, H * W < 2^31, B <= 65535.
 */
GKD_API gkd_status gkd_fuse_decode(const float* heat, const uint8_t* mask, long long mask_batch_stride, int B, int M,
                           int K, int H, int W, float* fused, float* xy, float* score, int32_t* idx,
                           uint8_t* valid, void* stream);

/*
 * Image preprocessing in front of the head ([CARD] Model section, Input
 * bullet: the ROI's longer side resized to 384 pixels, centre-padded to
 * 384 x 384 with the mean colour (124, 116, 104), ImageNet normalisation), for
 * B boxes of one image (one crop per detector box, the top-down use).
 *
 * For box b = (x0, y0, x1, y1) (image pixels, edge coordinates: pixel p spans
 * [p, p + 1)), s = canvas / max(x1 - x0, y1 - y0), ox = (canvas - (x1 - x0) s)/2,
 * oy likewise (not rounded). Canvas pixel (X, Y) is content iff its centre
 * (X + 0.5, Y + 0.5) lies in [ox, ox + (x1 - x0) s) x [oy, oy + (y1 - y0) s);
 * content takes the bilinear sample of the image at
 * (x0 + (X + 0.5 - ox)/s - 0.5, y0 + (Y + 0.5 - oy)/s - 0.5), each axis' two
 * taps clamped to the image, no antialiasing; other pixels take the pad colour.
 * Then out = (v / 255 - mean_c) / std_c, mean (0.485, 0.456, 0.406), std
 * (0.229, 0.224, 0.225). The page names no filter: this bilinear reading and
 * the unrounded pad offsets (the geometry of gkd_roi_to_image) are readings.
 * All arithmetic in fp64, rounded once to fp32.
 *
 *   img    [H][W][3] uint8 RGB, device memory
 *   boxes  [B][4] fp32 (x0, y0, x1, y1), device memory; a box with a
 *          non-positive or non-finite width or height gives an all-pad canvas
 *   out    [B][3][canvas][canvas] fp32 (channel-major)
 * Limits: 1 <= H, W <= 32768, B <= 65535, 1 <= canvas <= 4096 (384 for GKDT-L).
 */
GKD_API gkd_status gkd_preprocess(const uint8_t* img, int H, int W, const float* boxes, int B, int canvas,
                                  float* out, void* stream);

/*
 * ROI -> original-image coordinates of decoded keypoints ([CARD] Output
 * bullet, keypoints in the ROI's -1..1 space; Input bullet, the resize and
 * centre pad that this undoes): canvas pixel p = (u + 1) canvas / 2, then
 * x = x0 + (p_x - ox) / s, y = y0 + (p_y - oy) / s with s, ox, oy as in
 * gkd_preprocess. fp64 arithmetic, rounded once to fp32.
 *
 *   xy     [B][K][2] fp32 (as gkd_fuse_decode writes it), device memory
 *   boxes  [B][4] fp32 (x0, y0, x1, y1), device memory; a degenerate box gives NaN
 *   out    [B][K][2] fp32 image pixels (edge coordinates)
 * Rows of invalid keypoints are mapped like any other (xy = (0, 0) gives the
 * box centre); the caller keeps the valid flags.
 * Limits: B <= 65535, 1 <= K <= 65535, 1 <= canvas <= 4096.
 */
GKD_API gkd_status gkd_roi_to_image(const float* xy, const float* boxes, int B, int K, int canvas, float* out,
                                    void* stream);

/* Message for the last non-OK status returned on the calling thread ("" if none). */
GKD_API const char* gkd_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the calling device's error
 * word. Returns GKD_ERR_TIMEOUT if a kernel's bounded wait ran out since the
 * last check; GKD_ERR_CUDA if the stream reports a CUDA error or a kernel
 * recorded another failure (the tensor-core heatmap kernel refuses to run, and
 * writes nothing, if its tensor-memory allocation does not start at column 0);
 * else GKD_OK. There is one error word per device, shared by every launch of
 * this library on that device from any stream or thread. So the result covers
 * all of them, not only `stream`'s. A failure recorded by a kernel that is
 * still running elsewhere, between this call's read and its clear, is lost.
 * Call it when no other launch of the library is in flight on the device.
 */
GKD_API gkd_status gkd_check_device_error(void* stream);

/*
 * Upper bound, in milliseconds, on any single internal wait of the tensor-core
 * heatmap kernel (default 2000). Process-wide; applies to later launches.
 * Returns GKD_ERR_ARG for 0.
 */
GKD_API gkd_status gkd_set_wait_timeout_ms(unsigned int ms);

/*
 * Test hook: bit 0 makes the next gkd_heatmap launch on the bf16 path withhold
 * its upsample producers' first hand-off to the MMA warp, so the MMA warp's
 * bounded wait runs out and the kernel takes its timeout exit. The flags are
 * consumed (reset to 0) by that launch. Returns GKD_ERR_ARG for unknown bits.
 */
GKD_API gkd_status gkd_debug_set_flags(unsigned int flags);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
GKD_API int gkd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GKD_H_ */
