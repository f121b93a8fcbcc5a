// nf3.cuh -- the NF3 table format (MoLE page, 实验结果: a 3-bit table, e.g.
// NF3): the level table and the quantiser of one 64-element block, shared by
// the standalone quantiser (combine.cu) and the table build's quantising
// epilogue (build_tc.cu), so both produce the same codes bit for bit.
#pragma once

#include <cuda_bf16.h>
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

// The decision thresholds of a block with scale sc > 0, on the bf16 grid.
// The rule is c = #{k : RN(x / sc) > m_k} (RN: fp32 division, correctly
// rounded).  RN(q) > m_k holds exactly when q lies above b_k, the midpoint
// of m_k and the next fp32 value above it (q never equals b_k: b_k needs 25
// significant bits, x / sc for a bf16 x and an fp16 sc cannot have them), so
// for sc > 0 the rule is x > b_k * sc -- a product exact in fp64 (25 + 11
// bits).  x is a bf16 value, so x > P holds exactly when x > RD_bf16(P), the
// largest bf16 value not above P (rounded down to fp32, then to the bf16
// grid).  No division per element, and the same codes bit for bit.
__device__ __forceinline__ void nf3_thresholds(float sc, float (&t)[7]) {
  const float mid[7] = {MOLE_NF3_MIDPOINTS};
#pragma unroll
  for (int k = 0; k < 7; ++k) {
    const float m = mid[k];
    const float up = __int_as_float(__float_as_int(m) + (m > 0.f ? 1 : -1));  // next fp32 toward +inf
    const double b = 0.5 * ((double)m + (double)up);
    const float f = __double2float_rd(b * (double)sc);
    const uint32_t u = __float_as_uint(f);
    uint32_t r = u & 0xffff0000u;
    if ((u >> 31) != 0u && (u & 0xffffu) != 0u) r += 0x10000u;  // negative: away from zero is down
    t[k] = __uint_as_float(r);
  }
}

// The codes of both elements of a bf16 pair word xw (element 2i in the low
// half) against the thresholds, as bf16 pairs (t_k, t_k): seven packed
// compares (1.0 where x > t_k) added to 128.0 in bf16 -- 128 + c is exact
// for c <= 7 (the bf16 unit in [128, 256) is 1), and its low three bits are
// c.  Both x and the thresholds are bf16 values, so each compare is the
// exact comparison of nf3_code.  Returns lo | hi << 16.
__device__ __forceinline__ uint32_t nf3_code_pair(uint32_t xw, const __nv_bfloat162 (&t2)[7]) {
  const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&xw);
  __nv_bfloat162 c = __floats2bfloat162_rn(128.f, 128.f);
#pragma unroll
  for (int k = 0; k < 7; ++k) c = __hadd2(c, __hgt2(x, t2[k]));
  return *reinterpret_cast<const uint32_t*>(&c) & 0x00070007u;
}

// The thresholds as bf16 pairs (each t_k is a bf16 value, so exactly).
__device__ __forceinline__ void nf3_threshold_pairs(const float (&t)[7], __nv_bfloat162 (&t2)[7]) {
#pragma unroll
  for (int k = 0; k < 7; ++k) t2[k] = __floats2bfloat162_rn(t[k], t[k]);
}

// Code of one element x against the block's thresholds t (scale > 0).
__device__ __forceinline__ uint32_t nf3_code(float x, const float (&t)[7]) {
  uint32_t c = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) c += (x > t[k]) ? 1u : 0u;
  return c;
}

// Code c of element e at bits [3e, 3e+3) of the block's packed string.
__device__ __forceinline__ void nf3_put(uint32_t (&packed)[6], int e, uint32_t c) {
  const int bit = 3 * e;
  packed[bit >> 5] |= c << (bit & 31);
  if ((bit & 31) > 29) packed[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
}

// The block's fp16 scale: absmax, saturated at 65504, rounded to nearest even.
__device__ __forceinline__ __half nf3_scale(float amax) { return __float2half_rn(fminf(amax, 65504.f)); }

// One 64-element block (32 bf16 pairs, element 2i in the low half of xw[i]):
// amax -> fp16 scale (saturating, ties to even) -> the code of each element,
// the number of midpoints below RN(x / s) (nf3_thresholds) -> 3-bit code at
// bits [3e, 3e+3) of packed (24 bytes, little-endian).  Returns the scale's
// fp16 bits.
__device__ __forceinline__ uint16_t nf3_quantize_block(const uint32_t (&xw)[32], uint32_t (&packed)[6]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(xw[i])), fabsf(bf16_hi(xw[i]))));
  const __half s16 = nf3_scale(amax);
  const float sc = __half2float(s16);
#pragma unroll
  for (int i = 0; i < 6; ++i) packed[i] = 0u;
  if (sc == 0.f) {  // every code is the 0.0 level
#pragma unroll
    for (int e = 0; e < 64; ++e) nf3_put(packed, e, (uint32_t)kNf3ZeroCode);
    return __half_as_ushort(s16);
  }
  float t[7];
  nf3_thresholds(sc, t);
  __nv_bfloat162 t2[7];
  nf3_threshold_pairs(t, t2);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t c = nf3_code_pair(xw[i], t2);
    nf3_put(packed, 2 * i, c & 0xffffu);
    nf3_put(packed, 2 * i + 1, c >> 16);
  }
  return __half_as_ushort(s16);
}

}  // namespace
}  // namespace mole
