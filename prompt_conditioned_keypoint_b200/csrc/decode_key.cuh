// Peak keys for the decode fused into the heatmap kernels: one 64-bit key per
// (crop, prompt row) such that the largest key over all pixels is the first
// (lowest row-major index) maximal fused value, the rule of the two-kernel path
// (the peak of each prompt's heatmap, GKD_GGUF model card, Model section, Output
// bullet). Tiles of a crop reduce their candidates into one key with atomicMax.
//
//   bits 63..32  the value in an order-preserving unsigned form, -0 mapped to +0
//                (so +0 and -0 compare equal, as fp32 comparison does);
//   bits 31..1   0x7FFFFFFF - pixel index (equal values: the lowest index wins);
//   bit  0       the sign bit of a zero value (so the score keeps it).
// Key 0 means "no candidate": NaN values and pixels outside the heatmap never
// produce one.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace gkd {

__device__ __forceinline__ void peak_key(float f, uint32_t pixel, bool inside, uint32_t& hi, uint32_t& lo) {
  hi = 0;
  lo = 0;
  if (inside && f == f) {
    const uint32_t u = __float_as_uint(f);
    const bool zero = (u & 0x7FFFFFFFu) == 0;
    hi = zero ? 0x80000000u : ((u & 0x80000000u) ? ~u : (u | 0x80000000u));
    lo = ((0x7FFFFFFFu - pixel) << 1) | (zero ? (u >> 31) : 0u);
  }
}

// The warp's largest key (every lane gets it).
__device__ __forceinline__ unsigned long long warp_max_key(uint32_t hi, uint32_t lo) {
  const uint32_t whi = __reduce_max_sync(0xffffffffu, hi);
  const uint32_t wlo = __reduce_max_sync(0xffffffffu, hi == whi ? lo : 0u);
  return (static_cast<unsigned long long>(whi) << 32) | wlo;
}

}  // namespace gkd
