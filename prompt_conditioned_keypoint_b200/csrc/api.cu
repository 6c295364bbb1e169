// C ABI of libgkd (declared in include/gkd.h): host-side argument validation,
// device selection, per-device state and kernel launches. Checks that need no
// CUDA call (null pointers, sizes, dtypes, alignment) run first, so a bad call
// is rejected before the runtime is touched.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/gkd.h"
#include "gkd_internal.h"

namespace {

__device__ unsigned g_device_error_word;

// Peak keys of gkd_heatmap_decode_noalloc: one statically sized buffer per GPU
// that loads the library (1 MiB, held until the process exits), for callers
// that cannot hand the library any device memory of their own.
constexpr long long kNoAllocKeys = 131072;     // B * K at most
__device__ __align__(256) unsigned long long g_noalloc_keys[kNoAllocKeys];

thread_local std::string t_last_error;
std::atomic<unsigned> g_wait_timeout_ms{2000};
std::atomic<unsigned> g_debug_flags{0};

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  unsigned* err_word = nullptr;
  int num_sms = 0;
  unsigned long long* noalloc_keys = nullptr;   // device address of g_noalloc_keys on this device
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mutex;

gkd_status fail(gkd_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

gkd_status ok() {
  t_last_error.clear();
  return GKD_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device that owns `p` (a device or managed allocation); makes it current.
gkd_status use_device_of(const void* p, const char* name, int* dev_out) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(GKD_ERR_CUDA, "%s: cudaPointerGetAttributes failed: %s", name, cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(GKD_ERR_ARG, "%s must be a device pointer", name);
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != attr.device) {
    e = cudaSetDevice(attr.device);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "cudaSetDevice(%d) failed: %s", attr.device, cudaGetErrorString(e));
  }
  *dev_out = attr.device;
  return GKD_OK;
}

gkd_status check_same_device(const void* p, const char* name, int dev) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(GKD_ERR_CUDA, "%s: cudaPointerGetAttributes failed: %s", name, cudaGetErrorString(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(GKD_ERR_ARG, "%s must be a device pointer", name);
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
    return fail(GKD_ERR_ARG, "%s lives on device %d, expected device %d", name, attr.device, dev);
  return GKD_OK;
}

gkd_status device_state(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(GKD_ERR_ARG, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_error_word);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "error word lookup failed: %s", cudaGetErrorString(e));
    e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "SM count query failed: %s", cudaGetErrorString(e));
    // the host-side name g_noalloc_keys is only a stand-in: kernels need its
    // address on this device, looked up once here with the device current
    void* k = nullptr;
    e = cudaGetSymbolAddress(&k, g_noalloc_keys);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "static key buffer lookup failed: %s", cudaGetErrorString(e));
    d.noalloc_keys = static_cast<unsigned long long*>(k);
    d.err_word = static_cast<unsigned*>(p);
    d.ready = true;
  }
  *out = &d;
  return GKD_OK;
}

gkd_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

#define GKD_TRY(expr)                 \
  do {                                \
    gkd_status _s = (expr);           \
    if (_s != GKD_OK) return _s;      \
  } while (0)

}  // namespace

namespace gkd {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EncodeTiledFn>(nullptr);
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace gkd

extern "C" {

const char* gkd_last_error(void) { return t_last_error.c_str(); }

int gkd_version(void) { return 100; }

gkd_status gkd_set_wait_timeout_ms(unsigned int ms) {
  if (ms == 0) return fail(GKD_ERR_ARG, "timeout must be positive");
  g_wait_timeout_ms.store(ms);
  return ok();
}

gkd_status gkd_debug_set_flags(unsigned int flags) {
  if (flags & ~static_cast<unsigned>(gkd::kDbgSkipProducerArrive)) return fail(GKD_ERR_ARG, "unknown debug flag bits");
  g_debug_flags.store(flags);
  return ok();
}

gkd_status gkd_check_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "stream synchronize failed: %s", cudaGetErrorString(e));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GKD_ERR_CUDA, "cudaGetDevice failed");
  DeviceState* ds = nullptr;
  GKD_TRY(device_state(dev, &ds));
  unsigned word = 0, zero = 0;
  e = cudaMemcpy(&word, ds->err_word, sizeof word, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(ds->err_word, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "error word read failed: %s", cudaGetErrorString(e));
  if (word & gkd::kErrTimeout) return fail(GKD_ERR_TIMEOUT, "a kernel's bounded wait timed out (word 0x%x)", word);
  if (word & gkd::kErrBounds)
    return fail(GKD_ERR_CUDA, "a kernel's placement or bounds check failed; it did no work (word 0x%x)", word);
  if (word) return fail(GKD_ERR_CUDA, "device error word 0x%x", word);
  return ok();
}

gkd_status gkd_pool_prototypes(const void* support, gkd_dtype sdt, int B, int h, int w, int C, const float* kpts,
                               const uint8_t* kmask, int K, float sigma_px, float stride_px, float* proto,
                               long long proto_batch_stride, void* stream) {
  if (sdt != GKD_F32 && sdt != GKD_BF16) return fail(GKD_ERR_ARG, "sdt: unknown dtype %d", static_cast<int>(sdt));
  if (sdt != GKD_F32) return fail(GKD_ERR_DTYPE, "pooling takes fp32 support features");
  if (B < 0 || B > 65535) return fail(GKD_ERR_SHAPE, "B=%d out of range [0, 65535]", B);
  if (h < 1 || w < 1 || h > 256 || w > 256) return fail(GKD_ERR_SHAPE, "h=%d w=%d out of range [1, 256]", h, w);
  if (C < 8 || C % 8) return fail(GKD_ERR_SHAPE, "C=%d must be a positive multiple of 8", C);
  if (K < 1 || K > 128) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 128]", K);
  if (!(sigma_px > 0.f) || !(stride_px > 0.f)) return fail(GKD_ERR_ARG, "sigma and stride must be positive");
  if (proto_batch_stride < static_cast<long long>(K) * C)
    return fail(GKD_ERR_SHAPE, "proto_batch_stride=%lld < K*C", proto_batch_stride);
  if (B == 0) return ok();
  if (!support || !kpts || !kmask || !proto) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(support) || !aligned16(proto) || (proto_batch_stride * 4) % 16)
    return fail(GKD_ERR_ALIGN, "support/proto must be 16-byte aligned (and proto stride a multiple of 4)");
  if (reinterpret_cast<uintptr_t>(kpts) & 3u) return fail(GKD_ERR_ALIGN, "kpts must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(support, "support", &dev));
  GKD_TRY(check_same_device(kpts, "kpts", dev));
  GKD_TRY(check_same_device(kmask, "kmask", dev));
  GKD_TRY(check_same_device(proto, "proto", dev));
  DeviceState* ds = nullptr;
  GKD_TRY(device_state(dev, &ds));
  const char* why = "";
  const cudaError_t e = gkd::launch_pool_tc(
      static_cast<const float*>(support), B, h, w, C, kpts, kmask, K, sigma_px, stride_px, proto,
      proto_batch_stride, ds->err_word, static_cast<unsigned long long>(g_wait_timeout_ms.load()) * 1000000ull,
      ds->num_sms, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess && why[0]) return fail(GKD_ERR_CUDA, "pool: %s", why);
  return launched(e, "pool");
}

gkd_status gkd_norm_kernels(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C, float eps,
                            gkd_dtype out_dt, void* out, void* stream) {
  if (out_dt != GKD_F32 && out_dt != GKD_BF16) return fail(GKD_ERR_ARG, "out_dt: unknown dtype %d", static_cast<int>(out_dt));
  if (Bk < 0) return fail(GKD_ERR_SHAPE, "Bk=%d must be >= 0", Bk);
  if (M < 1 || M > 2) return fail(GKD_ERR_SHAPE, "M=%d must be 1 or 2", M);
  if (K < 1 || K > 128) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 128]", K);
  if (C < 8 || C % 8) return fail(GKD_ERR_SHAPE, "C=%d must be a positive multiple of 8", C);
  if (!(eps > 0.f)) return fail(GKD_ERR_ARG, "eps must be positive");
  const long long nrows = static_cast<long long>(Bk) * M * K;
  if (nrows >= (1ll << 31)) return fail(GKD_ERR_SHAPE, "too many rows");
  if (nrows == 0) return ok();
  if (!rows || !mask || !out) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(rows) || !aligned16(out)) return fail(GKD_ERR_ALIGN, "rows/out must be 16-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(rows, "rows", &dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(out, "out", dev));
  return launched(gkd::launch_norm(rows, mask, nrows, C, eps, out_dt == GKD_BF16, out,
                                   static_cast<cudaStream_t>(stream)),
                  "norm");
}

gkd_status gkd_norm_fuse_kernels(const float* rows, const uint8_t* mask, int Bk, int M, int K, int C, float eps,
                                 gkd_dtype out_dt, void* out, uint8_t* out_mask, void* stream) {
  if (out_dt != GKD_F32 && out_dt != GKD_BF16) return fail(GKD_ERR_ARG, "out_dt: unknown dtype %d", static_cast<int>(out_dt));
  if (Bk < 0) return fail(GKD_ERR_SHAPE, "Bk=%d must be >= 0", Bk);
  if (M < 1 || M > 2) return fail(GKD_ERR_SHAPE, "M=%d must be 1 or 2", M);
  if (K < 1 || K > 128) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 128]", K);
  if (C < 8 || C % 8) return fail(GKD_ERR_SHAPE, "C=%d must be a positive multiple of 8", C);
  if (!(eps > 0.f)) return fail(GKD_ERR_ARG, "eps must be positive");
  if (static_cast<long long>(Bk) * M * K >= (1ll << 31)) return fail(GKD_ERR_SHAPE, "too many rows");
  if (Bk == 0) return ok();
  if (!rows || !mask || !out || !out_mask) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(rows) || !aligned16(out)) return fail(GKD_ERR_ALIGN, "rows/out must be 16-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(rows, "rows", &dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(out, "out", dev));
  GKD_TRY(check_same_device(out_mask, "out_mask", dev));
  return launched(gkd::launch_norm_fuse(rows, mask, Bk, M, K, C, eps, out_dt == GKD_BF16, out, out_mask,
                                        static_cast<cudaStream_t>(stream)),
                  "norm_fuse");
}

}  // extern "C"

namespace {

// Argument checks shared by gkd_heatmap and gkd_heatmap_decode (no CUDA call).
gkd_status check_heatmap_args(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up, const void* kern,
                              gkd_dtype kdt, long long kern_batch_stride, const uint8_t* mask,
                              long long mask_batch_stride, int M, int K) {
  if (fdt != GKD_F32 && fdt != GKD_BF16) return fail(GKD_ERR_ARG, "fdt: unknown dtype %d", static_cast<int>(fdt));
  if (kdt != GKD_F32 && kdt != GKD_BF16) return fail(GKD_ERR_ARG, "kdt: unknown dtype %d", static_cast<int>(kdt));
  if (kdt == GKD_F32 && fdt != GKD_F32) return fail(GKD_ERR_DTYPE, "fp32 kernel rows need fp32 features");
  if (up != 4) return fail(GKD_ERR_SHAPE, "up=%d: only the 4x upsample is supported", up);
  if (B < 0 || B > 65535) return fail(GKD_ERR_SHAPE, "B=%d out of range [0, 65535]", B);
  if (h < 1 || w < 1 || h > 256 || w > 256) return fail(GKD_ERR_SHAPE, "h=%d w=%d out of range [1, 256]", h, w);
  if (C < 8 || C % 8) return fail(GKD_ERR_SHAPE, "C=%d must be a positive multiple of 8", C);
  if (M < 1 || M > 2) return fail(GKD_ERR_SHAPE, "M=%d must be 1 or 2", M);
  if (K < 1 || K > 128) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 128]", K);
  if (kdt == GKD_BF16 && M * ((K + 7) / 8 * 8) > 160)
    return fail(GKD_ERR_SHAPE, "M*ceil8(K)=%d exceeds the 160 accumulator columns", M * ((K + 7) / 8 * 8));
  if (kern_batch_stride < 0 || mask_batch_stride < 0) return fail(GKD_ERR_SHAPE, "batch strides must be >= 0");
  if (B == 0) return GKD_OK;
  if (!feat || !kern || !mask) return fail(GKD_ERR_ARG, "null tensor pointer");
  const int kelt = kdt == GKD_BF16 ? 2 : 4;
  if (!aligned16(feat) || !aligned16(kern) || (kern_batch_stride * kelt) % 16)
    return fail(GKD_ERR_ALIGN, "feat/kern must be 16-byte aligned and the kernel batch stride a 16-byte multiple");
  return GKD_OK;
}

// Fills the tensor-core kernel's arguments (device state looked up by the caller).
gkd::HeatmapTcArgs tc_args(const DeviceState* ds, gkd_dtype fdt, int B, int h, int w, int C, long long kern_batch_stride,
                           const uint8_t* mask, long long mask_batch_stride, int M, int K) {
  gkd::HeatmapTcArgs a{};
  a.mask = mask;
  a.mask_batch_stride = mask_batch_stride;
  a.B = B;
  a.h = h;
  a.w = w;
  a.C = C;
  a.M = M;
  a.K = K;
  a.feat_bf16 = fdt == GKD_BF16;
  a.kern_shared = kern_batch_stride == 0;
  a.err = ds->err_word;
  a.wait_limit_ns = static_cast<unsigned long long>(g_wait_timeout_ms.load()) * 1000000ull;
  a.debug_flags = g_debug_flags.exchange(0);
  return a;
}

// The three launches of the decode fused into the heatmap kernel: clear the
// per-(crop, row) keys, heatmap kernel in decode mode, keys -> outputs.
gkd_status enqueue_heatmap_decode(int dev, const void* feat, gkd_dtype fdt, int B, int h, int w, int C,
                                  const void* kern, gkd_dtype kdt, long long kern_batch_stride, const uint8_t* mask,
                                  long long mask_batch_stride, int M, int K, unsigned long long* keys, float* xy,
                                  float* score, int32_t* idx, uint8_t* valid, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(keys, 0, sizeof(unsigned long long) * static_cast<size_t>(B) * K, st);
  if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "scratch clear failed: %s", cudaGetErrorString(e));
  if (kdt == GKD_F32) {
    DeviceState* ds = nullptr;
    GKD_TRY(device_state(dev, &ds));
    e = gkd::launch_heatmap_f32(static_cast<const float*>(feat), B, h, w, C, static_cast<const float*>(kern),
                                kern_batch_stride, mask, mask_batch_stride, M, K, nullptr, keys, ds->num_sms, st);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "heatmap decode (fp32) launch failed: %s", cudaGetErrorString(e));
  } else {
    DeviceState* ds = nullptr;
    GKD_TRY(device_state(dev, &ds));
    gkd::HeatmapTcArgs a = tc_args(ds, fdt, B, h, w, C, kern_batch_stride, mask, mask_batch_stride, M, K);
    a.dec_keys = keys;
    const char* why = "";
    e = gkd::launch_heatmap_tc(a, feat, kern, kern_batch_stride, ds->num_sms, st, &why);
    if (e != cudaSuccess && why[0]) return fail(GKD_ERR_CUDA, "heatmap decode (bf16): %s", why);
    if (e != cudaSuccess) return fail(GKD_ERR_CUDA, "heatmap decode (bf16) launch failed: %s", cudaGetErrorString(e));
  }
  return launched(gkd::launch_finalize_keys(keys, mask, mask_batch_stride, B, M, K, 4 * h, 4 * w, xy, score, idx,
                                            valid, st),
                  "decode finalize");
}

}  // namespace

extern "C" {

gkd_status gkd_heatmap(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up, const void* kern,
                       gkd_dtype kdt, long long kern_batch_stride, const uint8_t* mask, long long mask_batch_stride,
                       int M, int K, float* heat, void* stream) {
  GKD_TRY(check_heatmap_args(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride, M, K));
  if (B == 0) return ok();
  if (!heat) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(heat)) return fail(GKD_ERR_ALIGN, "heat must be 16-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(feat, "feat", &dev));
  GKD_TRY(check_same_device(kern, "kern", dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(heat, "heat", dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DeviceState* ds = nullptr;
  GKD_TRY(device_state(dev, &ds));
  if (kdt == GKD_F32)
    return launched(gkd::launch_heatmap_f32(static_cast<const float*>(feat), B, h, w, C,
                                            static_cast<const float*>(kern), kern_batch_stride, mask,
                                            mask_batch_stride, M, K, heat, nullptr, ds->num_sms, st),
                    "heatmap (fp32)");
  gkd::HeatmapTcArgs a = tc_args(ds, fdt, B, h, w, C, kern_batch_stride, mask, mask_batch_stride, M, K);
  a.heat = heat;
  const char* why = "";
  cudaError_t e = gkd::launch_heatmap_tc(a, feat, kern, kern_batch_stride, ds->num_sms, st, &why);
  if (e != cudaSuccess && why[0]) return fail(GKD_ERR_CUDA, "heatmap (bf16): %s", why);
  return launched(e, "heatmap (bf16)");
}

gkd_status gkd_heatmap_decode(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up, const void* kern,
                              gkd_dtype kdt, long long kern_batch_stride, const uint8_t* mask,
                              long long mask_batch_stride, int M, int K, unsigned long long* scratch, float* xy,
                              float* score, int32_t* idx, uint8_t* valid, void* stream) {
  GKD_TRY(check_heatmap_args(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride, M, K));
  if (B == 0) return ok();
  if (!scratch || !xy || !score || !idx || !valid) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (reinterpret_cast<uintptr_t>(scratch) & 7u) return fail(GKD_ERR_ALIGN, "scratch must be 8-byte aligned");
  if ((reinterpret_cast<uintptr_t>(xy) | reinterpret_cast<uintptr_t>(score) | reinterpret_cast<uintptr_t>(idx)) & 3u)
    return fail(GKD_ERR_ALIGN, "xy/score/idx must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(feat, "feat", &dev));
  GKD_TRY(check_same_device(kern, "kern", dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(scratch, "scratch", dev));
  GKD_TRY(check_same_device(xy, "xy", dev));
  GKD_TRY(check_same_device(score, "score", dev));
  GKD_TRY(check_same_device(idx, "idx", dev));
  GKD_TRY(check_same_device(valid, "valid", dev));
  return enqueue_heatmap_decode(dev, feat, fdt, B, h, w, C, kern, kdt, kern_batch_stride, mask, mask_batch_stride,
                                M, K, scratch, xy, score, idx, valid, static_cast<cudaStream_t>(stream));
}

gkd_status gkd_fuse_decode(const float* heat, const uint8_t* mask, long long mask_batch_stride, int B, int M, int K,
                           int H, int W, float* fused, float* xy, float* score, int32_t* idx, uint8_t* valid,
                           void* stream) {
  if (B < 0 || B > 65535) return fail(GKD_ERR_SHAPE, "B=%d out of range [0, 65535]", B);
  if (M < 1 || M > 2) return fail(GKD_ERR_SHAPE, "M=%d must be 1 or 2", M);
  if (K < 1 || K > 65535) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 65535]", K);
  if (H < 1 || W < 1) return fail(GKD_ERR_SHAPE, "H=%d W=%d must be positive", H, W);
  const long long P = static_cast<long long>(H) * W;
  if (P % 4 || P >= (1ll << 31)) return fail(GKD_ERR_SHAPE, "H*W=%lld must be a multiple of 4 below 2^31", P);
  if (mask_batch_stride < 0) return fail(GKD_ERR_SHAPE, "mask_batch_stride must be >= 0");
  if (B == 0) return ok();
  if (!heat || !mask || !xy || !score || !idx || !valid) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(heat) || (fused && !aligned16(fused)))
    return fail(GKD_ERR_ALIGN, "heat/fused must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(xy) | reinterpret_cast<uintptr_t>(score) | reinterpret_cast<uintptr_t>(idx)) & 3u)
    return fail(GKD_ERR_ALIGN, "xy/score/idx must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(heat, "heat", &dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  if (fused) GKD_TRY(check_same_device(fused, "fused", dev));
  GKD_TRY(check_same_device(xy, "xy", dev));
  GKD_TRY(check_same_device(score, "score", dev));
  GKD_TRY(check_same_device(idx, "idx", dev));
  GKD_TRY(check_same_device(valid, "valid", dev));
  return launched(gkd::launch_fuse_decode(heat, mask, mask_batch_stride, B, M, K, H, W, fused, xy, score, idx, valid,
                                          static_cast<cudaStream_t>(stream)),
                  "fuse_decode");
}

gkd_status gkd_preprocess(const uint8_t* img, int H, int W, const float* boxes, int B, int canvas, float* out,
                          void* stream) {
  if (H < 1 || W < 1 || H > 32768 || W > 32768) return fail(GKD_ERR_SHAPE, "H=%d W=%d out of range [1, 32768]", H, W);
  if (B < 0 || B > 65535) return fail(GKD_ERR_SHAPE, "B=%d out of range [0, 65535]", B);
  if (canvas < 1 || canvas > 4096) return fail(GKD_ERR_SHAPE, "canvas=%d out of range [1, 4096]", canvas);
  if (B == 0) return ok();
  if (!img || !boxes || !out) return fail(GKD_ERR_ARG, "null tensor pointer");
  if ((reinterpret_cast<uintptr_t>(boxes) | reinterpret_cast<uintptr_t>(out)) & 3u)
    return fail(GKD_ERR_ALIGN, "boxes/out must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(img, "img", &dev));
  GKD_TRY(check_same_device(boxes, "boxes", dev));
  GKD_TRY(check_same_device(out, "out", dev));
  return launched(gkd::launch_preprocess(img, H, W, boxes, B, canvas, out, static_cast<cudaStream_t>(stream)),
                  "preprocess");
}

gkd_status gkd_roi_to_image(const float* xy, const float* boxes, int B, int K, int canvas, float* out, void* stream) {
  if (B < 0 || B > 65535) return fail(GKD_ERR_SHAPE, "B=%d out of range [0, 65535]", B);
  if (K < 1 || K > 65535) return fail(GKD_ERR_SHAPE, "K=%d out of range [1, 65535]", K);
  if (canvas < 1 || canvas > 4096) return fail(GKD_ERR_SHAPE, "canvas=%d out of range [1, 4096]", canvas);
  if (B == 0) return ok();
  if (!xy || !boxes || !out) return fail(GKD_ERR_ARG, "null tensor pointer");
  if ((reinterpret_cast<uintptr_t>(xy) | reinterpret_cast<uintptr_t>(boxes) | reinterpret_cast<uintptr_t>(out)) & 3u)
    return fail(GKD_ERR_ALIGN, "xy/boxes/out must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(xy, "xy", &dev));
  GKD_TRY(check_same_device(boxes, "boxes", dev));
  GKD_TRY(check_same_device(out, "out", dev));
  return launched(gkd::launch_roi_to_image(xy, boxes, B, K, canvas, out, static_cast<cudaStream_t>(stream)),
                  "roi_to_image");
}

gkd_status gkd_heatmap_contract_first(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                                     const void* kern, long long kern_batch_stride, const uint8_t* mask,
                                     long long mask_batch_stride, int M, int K, float* scratch, float* heat,
                                     void* stream) {
  GKD_TRY(check_heatmap_args(feat, fdt, B, h, w, C, up, kern, GKD_BF16, kern_batch_stride, mask, mask_batch_stride,
                             M, K));
  if (B == 0) return ok();
  if (!scratch || !heat) return fail(GKD_ERR_ARG, "null tensor pointer");
  if (!aligned16(heat) || (reinterpret_cast<uintptr_t>(scratch) & 3u))
    return fail(GKD_ERR_ALIGN, "heat must be 16-byte aligned and scratch 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(feat, "feat", &dev));
  GKD_TRY(check_same_device(kern, "kern", dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(scratch, "scratch", dev));
  GKD_TRY(check_same_device(heat, "heat", dev));
  DeviceState* ds = nullptr;
  GKD_TRY(device_state(dev, &ds));
  gkd::ContractArgs a{};
  a.mask = mask;
  a.mask_batch_stride = mask_batch_stride;
  a.G = scratch;
  a.B = B;
  a.h = h;
  a.w = w;
  a.C = C;
  a.M = M;
  a.K = K;
  a.feat_bf16 = fdt == GKD_BF16;
  a.kern_shared = kern_batch_stride == 0;
  a.err = ds->err_word;
  a.wait_limit_ns = static_cast<unsigned long long>(g_wait_timeout_ms.load()) * 1000000ull;
  const char* why = "";
  cudaError_t e = gkd::launch_contract_first(a, feat, kern, kern_batch_stride, heat, static_cast<cudaStream_t>(stream),
                                             &why);
  if (e != cudaSuccess && why[0]) return fail(GKD_ERR_CUDA, "contract-first heatmap: %s", why);
  return launched(e, "contract-first heatmap");
}

gkd_status gkd_heatmap_decode_noalloc(const void* feat, gkd_dtype fdt, int B, int h, int w, int C, int up,
                                      const void* kern, gkd_dtype kdt, long long kern_batch_stride,
                                      const uint8_t* mask, long long mask_batch_stride, int M, int K, float* xy,
                                      float* score, int32_t* idx, uint8_t* valid, void* stream) {
  GKD_TRY(check_heatmap_args(feat, fdt, B, h, w, C, up, kern, kdt, kern_batch_stride, mask, mask_batch_stride, M, K));
  if (static_cast<long long>(B) * K > kNoAllocKeys)
    return fail(GKD_ERR_SHAPE, "B*K=%lld exceeds the %lld peak keys of the static buffer (use gkd_heatmap_decode)",
                static_cast<long long>(B) * K, kNoAllocKeys);
  if (B == 0) return ok();
  if (!xy || !score || !idx || !valid) return fail(GKD_ERR_ARG, "null tensor pointer");
  if ((reinterpret_cast<uintptr_t>(xy) | reinterpret_cast<uintptr_t>(score) | reinterpret_cast<uintptr_t>(idx)) & 3u)
    return fail(GKD_ERR_ALIGN, "xy/score/idx must be 4-byte aligned");
  int dev = 0;
  GKD_TRY(use_device_of(feat, "feat", &dev));
  GKD_TRY(check_same_device(kern, "kern", dev));
  GKD_TRY(check_same_device(mask, "mask", dev));
  GKD_TRY(check_same_device(xy, "xy", dev));
  GKD_TRY(check_same_device(score, "score", dev));
  GKD_TRY(check_same_device(idx, "idx", dev));
  GKD_TRY(check_same_device(valid, "valid", dev));
  DeviceState* ds = nullptr;
  GKD_TRY(device_state(dev, &ds));
  return enqueue_heatmap_decode(dev, feat, fdt, B, h, w, C, kern, kdt, kern_batch_stride, mask, mask_batch_stride,
                                M, K, ds->noalloc_keys, xy, score, idx, valid, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
