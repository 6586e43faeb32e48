// The MX quantisation rule for one block of 32 bf16 values (the OCP
// Microscaling formats, MXFP8 with E4M3 elements; "Mixture-of-Kittens: A MoE
// Megakernel for GB300 NVL72", section 5): shared by the quantising dispatch
// kernels and by the MXFP8 GEMM1's landed dispatch.
//
// amax = max |v|; the shared exponent e = floor(log2 amax) - 8 (8: the
// exponent of E4M3's largest normal, 448), clamped to [-127, 127], -127 for an
// all-zero block; the scale is stored as the E8M0 code e + 127 and each
// element as E4M3(v * 2^-e), nearest-even with magnitudes above 448 clamped to
// 448 (CUDA's saturating fp32 -> E4M3 pair conversion). floor(log2 amax) comes
// straight from the bf16 exponent bits (subnormal inputs included), and
// v * 2^-e is exact, so the codes depend on nothing but the inputs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {
namespace mx {

// floor(log2 |v|) of a non-zero bf16 magnitude (sign bit clear), exactly.
__device__ __forceinline__ int bf16_floor_log2(uint32_t mag) {
  const int ef = static_cast<int>(mag >> 7);
  if (ef != 0) return ef - 127;
  return -134 + (32 - __clz(mag));  // subnormal: 2^-133 * mantissa
}

// One 32-element block: 4 x 16 bytes of bf16 in, 2 x 16 bytes of E4M3 codes
// and one E8M0 scale code out.
__device__ __forceinline__ void mx_block(const uint4 (&in)[4], uint4 (&out)[2], uint8_t& scale) {
  uint32_t amax = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t w[4] = {in[v].x, in[v].y, in[v].z, in[v].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = max(amax, w[i] & 0x7FFFu);
      amax = max(amax, (w[i] >> 16) & 0x7FFFu);
    }
  }
  int e = -127;
  if (amax != 0) e = max(-127, min(127, bf16_floor_log2(amax) - 8));
  scale = static_cast<uint8_t>(e + 127);
  // 2^-e as a normal fp32 (bf16 magnitudes keep e <= 119); the products are
  // exact except when they fall far below E4M3's smallest step, where the
  // code is a signed zero either way
  const float inv = __int_as_float((127 - e) << 23);
  uint32_t codes[8];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t w[4] = {in[v].x, in[v].y, in[v].z, in[v].w};
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      uint32_t packed = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // one bf16 pair -> two code bytes (low element first)
        const uint32_t word = w[i + h];
        const float2 f = make_float2(__uint_as_float(word << 16) * inv,
                                     __uint_as_float(word & 0xFFFF0000u) * inv);
        const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
        packed |= static_cast<uint32_t>(c2) << (16 * h);
      }
      codes[v * 2 + i / 2] = packed;
    }
  }
  out[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  out[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
}

}  // namespace mx
}  // namespace moe
