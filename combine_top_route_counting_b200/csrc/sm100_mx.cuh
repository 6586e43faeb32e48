// Inline-PTX wrappers for the block-scaled (MXFP8) tcgen05 path: the
// instruction descriptor of kind::mxf8f6f4 with E8M0 scales, the unswizzled
// shared-memory descriptor of tcgen05.cp, the CTA-pair scale copy into TMEM
// and the CTA-pair block-scaled MMA. Used by expert_ffn_mx.cu only.
#pragma once

#include "sm100.cuh"

namespace moe {
namespace sm100 {

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A and B E4M3
// (format code 0), both K-major, E8M0 scales, fp32 D, shape M x N, dense K = 32.
// a_sf_id / b_sf_id pick the byte of each 32-bit TMEM scale cell that this
// instruction's 32-element K block uses.
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3(uint32_t M, uint32_t N, uint32_t a_sf_id,
                                                       uint32_t b_sf_id) {
  return (b_sf_id << 4)       // B scale-factor id
         | ((N >> 3) << 17)   // N / 8
         | (1u << 23)         // scale format: E8M0
         | ((M >> 4) << 24)   // M / 16
         | (a_sf_id << 29);   // A scale-factor id
}

// Shared-memory descriptor of an unswizzled K-major column of 8-row x 16-byte
// core matrices (rows 16 bytes apart, consecutive core matrices `sbo` bytes
// apart, one core matrix along K): the source operand of tcgen05.cp.
__device__ __forceinline__ uint64_t smem_desc_noswz(uint32_t saddr, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);  // layout 0: none
}

// CTA pair: copy 32 rows x 128 bits of each CTA's shared memory (descriptor
// sdesc, same offset in both) into that CTA's TMEM lanes 0-31, columns
// taddr .. taddr+3, replicated into all four lane quarters. Issued by one
// thread of the leader; ordered before the same thread's later tcgen05.mma.
__device__ __forceinline__ void tc_cp_pair_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= (A . 2^sfA) x (B . 2^sfB) over the CTA pair, E4M3 operands, one
// E8M0 scale per row (A) or column (B) per 32 K values read from TMEM at tsfa /
// tsfb (bits 31:30 of each address name the byte, as in the descriptor).
__device__ __forceinline__ void tc_mma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

}  // namespace sm100
}  // namespace moe
