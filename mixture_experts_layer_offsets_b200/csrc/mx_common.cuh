// mx_common.cuh -- device helpers of the MXFP8 format shared by the quantisers and the
// GEMM epilogues that write MXFP8 operands.
//
// Page: "Ai2 Olmo-core 3：MoE训练吞吐量提升2.7倍的秘诀" (kongchang.com), section
// 吞吐量数字的边界条件: blocks of 32 elements share one scale.  Rule (OCP MX conversion):
// e = floor(log2(amax)) - 8, clamped to [-127, 127] (amax 0 -> -127); scale byte e + 127;
// element = E4M3 round-to-nearest-even of v * 2^-e with saturation at 448, sign of v kept.
#pragma once

#include <stdint.h>

namespace moe {

// floor(log2(amax)) - 8 from the fp32 exponent bits (exact, subnormals included),
// clamped to the E8M0 range.
__device__ __forceinline__ int block_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int ex = (int)((bits >> 23) & 0xFF);
  int fl;
  if (ex == 0) {
    const uint32_t man = bits & 0x7FFFFF;
    if (man == 0) return -127;
    fl = -149 + (31 - __clz(man));
  } else {
    fl = ex - 127;
  }
  return min(max(fl - 8, -127), 127);
}

// 2^-e as an fp32 (e <= 119 for any finite fp32 amax, so 2^-e is normal).
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

// Two E4M3 codes (hi in the upper byte): the hardware conversion rounds to nearest even,
// saturates at +-448 and keeps the sign, a negative value that rounds to zero included
// (code 0x80).
__device__ __forceinline__ uint32_t e4m3_pair(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- scale atoms
// The block-scaled MMA takes its E8M0 scales from TMEM, which each pipeline stage fills
// from a 512-byte shared-memory atom: 128 rows (of M or N) x 4 blocks of 32 along K, the
// scale of row r and block kb at byte (r % 32) * 16 + (r / 32) * 4 + kb.  Inside the FFN
// every scale lives in global memory as such atoms, in the order in which the grouped
// GEMM consumes them, so that one bulk copy per operand and stage fetches it.
__device__ __forceinline__ int atom_byte(int r, int kb) {
  return (r & 31) * 16 + ((r >> 5) & 3) * 4 + kb;
}

}  // namespace moe
