// nf3.cuh -- the NF3 table format (MoLE page, 实验结果: a 3-bit table, e.g.
// NF3): the level table and the quantiser of one 64-element block, shared by
// the standalone quantiser (combine.cu) and the table build's quantising
// epilogue (build_tc.cu), so both produce the same codes bit for bit.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace mole {
namespace {

// NormalFloat k=3 levels (QLoRA construction, rounded to fp16; ascending,
// index 3 is 0.0) and the fp32 midpoints of adjacent levels.
constexpr uint16_t kNf3Levels[8] = {0xbc00, 0xb848, 0xb3e7, 0x0000, 0x31de, 0x361d, 0x38fc, 0x3c00};
#define MOLE_NF3_MIDPOINTS -0x1.89p-1f, -0x1.907p-2f, -0x1.f9cp-4f, 0x1.778p-4f, 0x1.218p-2f, 0x1.015p-1f, 0x1.9f8p-1f
constexpr float kNf3Mid[7] = {MOLE_NF3_MIDPOINTS};
constexpr int kNf3ZeroCode = 3;

// One 64-element block (32 bf16 pairs, element 2i in the low half of xw[i]),
// all in IEEE fp32: amax -> fp16 scale (saturating, ties to even) -> correctly
// rounded x / s -> number of midpoints below -> 3-bit code at bits [3e, 3e+3)
// of packed (24 bytes, little-endian).  Returns the scale's fp16 bits.
__device__ __forceinline__ uint16_t nf3_quantize_block(const uint32_t (&xw)[32], uint32_t (&packed)[6]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(xw[i])), fabsf(bf16_hi(xw[i]))));
  const __half s16 = __float2half_rn(fminf(amax, 65504.f));
  const float sc = __half2float(s16);
  const float mid[7] = {MOLE_NF3_MIDPOINTS};
#pragma unroll
  for (int i = 0; i < 6; ++i) packed[i] = 0u;
#pragma unroll
  for (int e = 0; e < 64; ++e) {
    const float x = (e & 1) ? bf16_hi(xw[e >> 1]) : bf16_lo(xw[e >> 1]);
    uint32_t c;
    if (sc == 0.f) {
      c = kNf3ZeroCode;
    } else {
      const float y = __fdiv_rn(x, sc);
      c = 0;
#pragma unroll
      for (int k = 0; k < 7; ++k) c += (y > mid[k]) ? 1u : 0u;
    }
    const int bit = 3 * e;
    packed[bit >> 5] |= c << (bit & 31);
    if ((bit & 31) > 29) packed[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
  }
  return __half_as_ushort(s16);
}

}  // namespace
}  // namespace mole
