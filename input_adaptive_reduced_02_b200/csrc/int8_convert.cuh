// Exact int8 -> f32 / bf16 conversions for the INT8-weight kernels (row
// norms, pack, gather-GEMV), on the integer and FP32 pipes.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace rmm {

// Four signed bytes -> f32, exactly, on the integer and FP32 pipes (the
// int-to-float conversion unit issues at a fraction of their rate). With its
// sign bit flipped, the byte of a value v in [-128, 127] reads v + 128 in
// [0, 255]; placed in the low mantissa bits of 2^23 it makes the float
// 2^23 + v + 128, and subtracting 2^23 + 128 leaves v. Every quantity is an
// integer below 2^24, so the subtraction is exact.
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float& f0, float& f1, float& f2, float& f3) {
  const uint32_t u = w ^ 0x80808080u;
  constexpr uint32_t kTwo23 = 0x4B000000u;  // 2^23
  constexpr float kBias = 8388736.0f;       // 2^23 + 128
  f0 = __uint_as_float(__byte_perm(u, kTwo23, 0x7650)) - kBias;
  f1 = __uint_as_float(__byte_perm(u, kTwo23, 0x7651)) - kBias;
  f2 = __uint_as_float(__byte_perm(u, kTwo23, 0x7652)) - kBias;
  f3 = __uint_as_float(__byte_perm(u, kTwo23, 0x7653)) - kBias;
}

// f32 pair whose values are exact in bf16 (at most 8 significant bits, e.g.
// integers of magnitude <= 256) -> bf16x2: the upper halves, no rounding needed.
__device__ __forceinline__ uint32_t pack_bf16x2_exact(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
}

}  // namespace rmm
