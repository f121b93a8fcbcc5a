// combine.cu -- fused router + softmax + direct-addressed gather + gate-weighted
// sum over the lookup table (MoLE page, 训练阶段 and 推理阶段: the router sees the
// previous layer's hidden state, every routed expert is active, and each
// token's expert outputs are fetched from the table by its token id).
//
//   out[t, :] = sum_j softmax(h[t] . Wr)_j  LUT[ids[t], j, :]
//
// One persistent CTA (256 threads) walks token tiles of up to 16 tokens:
//   1. router: the tile's logits z[16, N] = h_tile . Wr.  For bf16 inputs this
//      is a tensor-core contraction (mma.sync m16n8k16, fp32 accumulate) with
//      the D dimension split across the 8 warps; Wr is staged once per CTA in
//      shared memory, transposed to [N][D] so each B fragment is one 8-byte
//      load.  h fragments are loaded straight from global memory.  The k-slot
//      order inside a 16-wide step is permuted (slots 2c,2c+1 <- d+4c+0,1 and
//      2c+8,2c+9 <- d+4c+2,3) so that each lane's A and B pieces are
//      contiguous; a dot product does not depend on that order.
//   2. softmax over the N experts of each token (max-subtracted, fp32), gates
//      kept in shared memory.
//   3. gather + combine: each thread owns one 16-byte vector of D of one token
//      and issues the N row loads LUT[id, j, vec] back to back (N x 16 B in
//      flight per thread) before the fp32 FMAs; rows stream from HBM through
//      registers (no shared-memory staging, which would double the on-chip
//      traffic per byte).
#include <math.h>

#include "common.cuh"

namespace mole {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTileMax = 16;  // rows of the m16n8k16 router MMA

enum TableKind { kTableBf16 = 0, kTableF32 = 1, kTableNf3 = 2 };

// ---- NF3 level table (NormalFloat k=3 levels, QLoRA construction, rounded to
// fp16; ascending, index 3 is 0.0) and the fp32 midpoints of adjacent levels.
constexpr uint16_t kNf3Levels[8] = {0xbc00, 0xb848, 0xb3e7, 0x0000, 0x31de, 0x361d, 0x38fc, 0x3c00};
#define MOLE_NF3_MIDPOINTS -0x1.89p-1f, -0x1.907p-2f, -0x1.f9cp-4f, 0x1.778p-4f, 0x1.218p-2f, 0x1.015p-1f, 0x1.9f8p-1f
constexpr float kNf3Mid[7] = {MOLE_NF3_MIDPOINTS};
constexpr int kNf3ZeroCode = 3;

// Byte planes of the fp16 levels, for prmt lookups: plane[k] holds byte k of
// level k (low bytes in kLoBytes*, high bytes in kHiBytes*).
constexpr uint32_t byte_plane(int first, int shift) {
  return ((uint32_t)((kNf3Levels[first + 0] >> shift) & 0xff)) |
         ((uint32_t)((kNf3Levels[first + 1] >> shift) & 0xff) << 8) |
         ((uint32_t)((kNf3Levels[first + 2] >> shift) & 0xff) << 16) |
         ((uint32_t)((kNf3Levels[first + 3] >> shift) & 0xff) << 24);
}
constexpr uint32_t kLoBytes0 = byte_plane(0, 0), kLoBytes1 = byte_plane(4, 0);
constexpr uint32_t kHiBytes0 = byte_plane(0, 8), kHiBytes1 = byte_plane(4, 8);

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared-memory carve-up of one CTA (NP = padded expert count, 8 * NT).
struct Smem {
  uint16_t* wrt;  // [NP][D + 8] bf16 Wr^T (bf16 router only)
  float* part;    // [kWarps][kTileMax][NP] router partial sums
  float* gates;   // [kTileMax][NP]
  int* tok_id;    // [kTileMax]
};

template <bool kBf16Router, int NP>
__host__ __device__ constexpr size_t smem_bytes_for(int D) {
  return (kBf16Router ? (size_t)NP * (D + 8) * 2 : 0) + (size_t)kWarps * kTileMax * NP * 4 +
         (size_t)kTileMax * NP * 4 + (size_t)kTileMax * 4;
}

template <bool kBf16Router, int NP>
__device__ __forceinline__ Smem carve(uint8_t* base, int D) {
  Smem s;
  size_t off = 0;
  s.wrt = reinterpret_cast<uint16_t*>(base);
  if (kBf16Router) off += (size_t)NP * (D + 8) * 2;
  s.part = reinterpret_cast<float*>(base + off);
  off += (size_t)kWarps * kTileMax * NP * 4;
  s.gates = reinterpret_cast<float*>(base + off);
  off += (size_t)kTileMax * NP * 4;
  s.tok_id = reinterpret_cast<int*>(base + off);
  return s;
}

// Stage Wr^T in shared memory: wrt[j][d] = Wr[d][j] (bf16), zero rows j >= N.
// Loads are issued in batches of 8 per thread before their stores so their
// latencies overlap (a dependent load per element would serialise them).
template <int NP, int kNThreads>
__device__ __forceinline__ void stage_wrt(uint16_t* wrt, const uint16_t* __restrict__ wr, int N, int D) {
  const int ldw = D + 8;
  if (N == NP && (reinterpret_cast<uintptr_t>(wr) & 15u) == 0) {
    // 16-byte loads of 8 experts of one row d, 16 per thread in flight
    const int total8 = D * NP / 8;
    for (int base = threadIdx.x; base < total8; base += kNThreads * 16) {
      uint4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = base + u * kNThreads;
        if (i < total8) v[u] = __ldg(reinterpret_cast<const uint4*>(wr) + i);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = base + u * kNThreads;
        if (i < total8) {
          const int d = (i * 8) / NP, j0 = (i * 8) % NP;
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            wrt[(j0 + 2 * e) * ldw + d] = (uint16_t)(w[e] & 0xffffu);
            wrt[(j0 + 2 * e + 1) * ldw + d] = (uint16_t)(w[e] >> 16);
          }
        }
      }
    }
    return;
  }
  const int total = D * NP;
  for (int base = threadIdx.x; base < total; base += kNThreads * 8) {
    uint16_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * kNThreads;
      const int d = i / NP, j = i - d * NP;
      v[u] = (i < total && j < N) ? __ldg(wr + (int64_t)d * N + j) : (uint16_t)0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * kNThreads;
      if (i < total) {
        const int d = i / NP, j = i - d * NP;
        wrt[j * ldw + d] = v[u];
      }
    }
  }
}

// Router + softmax for one tile of `rows` tokens starting at t0.  On return
// (after a __syncthreads) s.gates[r][j] and s.tok_id[r] are valid for r < rows.
template <bool kBf16Router, int NT>
__device__ __forceinline__ void router_tile(const Smem& s, const int32_t* __restrict__ ids,
                                            const void* __restrict__ h_, const void* __restrict__ Wr_,
                                            int64_t t0, int rows, int N, int D) {
  constexpr int NP = 8 * NT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (kBf16Router) {
    constexpr int KB = 16;  // k-steps whose A fragments are fetched before their MMAs
    const uint16_t* h = static_cast<const uint16_t*>(h_);
    const int g = lane >> 2, c = lane & 3, ldw = D + 8;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const bool ok0 = g < rows, ok1 = g + 8 < rows;
    const uint16_t* h0 = h + (t0 + (ok0 ? g : 0)) * (int64_t)D + 4 * c;
    const uint16_t* h1 = h + (t0 + (ok1 ? g + 8 : 0)) * (int64_t)D + 4 * c;
    const uint16_t* w = s.wrt + g * ldw + 4 * c;
    const int ksteps = D >> 4;
    for (int kb = warp; kb < ksteps; kb += kWarps * KB) {
      uint2 a0[KB], a1[KB];
#pragma unroll
      for (int i = 0; i < KB; ++i) {
        const int ks = kb + i * kWarps;
        const bool in = ks < ksteps;
        a0[i] = (in && ok0) ? __ldg(reinterpret_cast<const uint2*>(h0 + (ks << 4))) : make_uint2(0u, 0u);
        a1[i] = (in && ok1) ? __ldg(reinterpret_cast<const uint2*>(h1 + (ks << 4))) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < KB; ++i) {
        const int ks = kb + i * kWarps;
        if (ks < ksteps) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = *reinterpret_cast<const uint2*>(w + nt * 8 * ldw + (ks << 4));
            mma_16816(acc[nt], a0[i].x, a1[i].x, a0[i].y, a1[i].y, b.x, b.y);
          }
        }
      }
    }
    float* pw = s.part + warp * kTileMax * NP;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      pw[g * NP + nt * 8 + 2 * c] = acc[nt][0];
      pw[g * NP + nt * 8 + 2 * c + 1] = acc[nt][1];
      pw[(g + 8) * NP + nt * 8 + 2 * c] = acc[nt][2];
      pw[(g + 8) * NP + nt * 8 + 2 * c + 1] = acc[nt][3];
    }
  } else {
    // fp32 router on CUDA cores: one warp per token row, lanes split D.
    const float* h = static_cast<const float*>(h_);
    const float* Wr = static_cast<const float*>(Wr_);
    for (int r = warp; r < kTileMax; r += kWarps) {
      float p[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) p[j] = 0.f;
      if (r < rows) {
        const float* hr = h + (t0 + r) * (int64_t)D;
        for (int d = lane; d < D; d += 32) {
          const float hv = __ldg(hr + d);
#pragma unroll
          for (int j = 0; j < NP; ++j)
            if (j < N) p[j] = fmaf(hv, __ldg(Wr + (int64_t)d * N + j), p[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        float v = p[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        p[j] = v;
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < NP; ++j) s.part[r * NP + j] = p[j];
      }
    }
  }
  __syncthreads();
  // tok_id is written only now: before this barrier, threads still finishing
  // the previous tile's gather may be reading it.
  if (tid < rows) s.tok_id[tid] = __ldg(ids + t0 + tid);

  // softmax: NP lanes per token row (NP in {8, 16, 32})
  constexpr int RPW = 32 / NP;
  const int sub = lane / NP, jl = lane % NP;
  for (int rb = warp * RPW; rb < rows; rb += kWarps * RPW) {
    const int r = rb + sub;
    const bool act = r < rows;
    float z = 0.f;
    if (act) {
      if (kBf16Router) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) z += s.part[(w * kTileMax + r) * NP + jl];
      } else {
        z = s.part[r * NP + jl];
      }
    }
    const bool valid = act && jl < N;
    float m = valid ? z : -INFINITY;
#pragma unroll
    for (int off = NP / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float e = valid ? expf(z - m) : 0.f;
    float sum = e;
#pragma unroll
    for (int off = NP / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (act) s.gates[r * NP + jl] = valid ? e / sum : 0.f;
  }
  __syncthreads();
}

// Which (token row, unit) pairs of a tile this thread handles, for `per_tok`
// units per token: with fewer units per token than threads, several tokens
// are covered per pass; computed once per thread, so the gather loop does no
// division.
struct UnitMap {
  int r0, rstep, v0, vstep;
  __device__ __forceinline__ UnitMap(int per_tok) {
    const int tid = threadIdx.x;
    if (per_tok >= kThreads) {
      r0 = 0;
      rstep = 1;
      v0 = tid;
      vstep = kThreads;
    } else {
      const int rp = kThreads / per_tok;
      v0 = tid % per_tok;
      r0 = tid / per_tok;
      rstep = rp;
      vstep = per_tok;
      if (r0 >= rp) r0 = kTileMax;  // spare threads: no unit
    }
  }
};

__device__ __forceinline__ void store_nan(float* o, int n) {
  for (int i = 0; i < n; i += 4) __stcs(reinterpret_cast<float4*>(o + i), make_float4(NAN, NAN, NAN, NAN));
}

__device__ __forceinline__ void load_gates(const float* gr, float* g, int n) {
  for (int i = 0; i < n; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(gr + i);
    g[i] = v.x;
    g[i + 1] = v.y;
    g[i + 2] = v.z;
    g[i + 3] = v.w;
  }
}

// Gather + combine of one tile from a bf16 table: unit = (token, 8-wide
// vector).  All N row loads of a unit are issued before its first FMA; with
// an exact expert count there is no predication at all.
template <int NT, bool kExactN>
__device__ __forceinline__ void combine_tile_bf16(const Smem& s, const UnitMap& um,
                                                  const uint16_t* __restrict__ lut, int64_t V, int N,
                                                  int D, int64_t t0, int rows, float* __restrict__ out,
                                                  unsigned* err) {
  constexpr int NP = 8 * NT;
  constexpr int CH = NP < 16 ? NP : 16;  // rows in flight per batch (64 registers)
  const int DV = D >> 3;
  for (int r = um.r0; r < rows; r += um.rstep) {
    const int id = s.tok_id[r];
    float g[NP];
    load_gates(s.gates + r * NP, g, NP);
    for (int v = um.v0; v < DV; v += um.vstep) {
      float* o = out + (t0 + r) * (int64_t)D + v * 8;
      if (id < 0 || (int64_t)id >= V) {
        if (v == 0) atomicOr(err, kErrIndex);
        store_nan(o, 8);
        continue;
      }
      const uint4* src = reinterpret_cast<const uint4*>(lut + (int64_t)id * N * D) + v;
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = 0.f;
#pragma unroll
      for (int j0 = 0; j0 < NP; j0 += CH) {
        uint4 x[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const int jj = kExactN ? j0 + j : min(j0 + j, N - 1);  // padded experts re-read a valid row
          x[j] = __ldg(src + (int64_t)jj * DV);
        }
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          if (kExactN || j0 + j < N) {
            const float gj = g[j0 + j];
            a[0] = fmaf(gj, bf16_lo(x[j].x), a[0]);
            a[1] = fmaf(gj, bf16_hi(x[j].x), a[1]);
            a[2] = fmaf(gj, bf16_lo(x[j].y), a[2]);
            a[3] = fmaf(gj, bf16_hi(x[j].y), a[3]);
            a[4] = fmaf(gj, bf16_lo(x[j].z), a[4]);
            a[5] = fmaf(gj, bf16_hi(x[j].z), a[5]);
            a[6] = fmaf(gj, bf16_lo(x[j].w), a[6]);
            a[7] = fmaf(gj, bf16_hi(x[j].w), a[7]);
          }
        }
      }
      __stcs(reinterpret_cast<float4*>(o), make_float4(a[0], a[1], a[2], a[3]));
      __stcs(reinterpret_cast<float4*>(o + 4), make_float4(a[4], a[5], a[6], a[7]));
    }
  }
}

// Gather + combine of one tile from an fp32 table: unit = (token, 4-wide vector).
template <int NT, bool kExactN>
__device__ __forceinline__ void combine_tile_f32(const Smem& s, const UnitMap& um,
                                                 const float* __restrict__ lut, int64_t V, int N, int D,
                                                 int64_t t0, int rows, float* __restrict__ out,
                                                 unsigned* err) {
  constexpr int NP = 8 * NT;
  const int DV = D >> 2;
  for (int r = um.r0; r < rows; r += um.rstep) {
    const int id = s.tok_id[r];
    float g[NP];
    load_gates(s.gates + r * NP, g, NP);
    for (int v = um.v0; v < DV; v += um.vstep) {
      float* o = out + (t0 + r) * (int64_t)D + v * 4;
      if (id < 0 || (int64_t)id >= V) {
        if (v == 0) atomicOr(err, kErrIndex);
        store_nan(o, 4);
        continue;
      }
      const float4* src = reinterpret_cast<const float4*>(lut + (int64_t)id * N * D) + v;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        if (kExactN || j < N) {
          const float4 x = __ldg(src + (int64_t)j * DV);
          a.x = fmaf(g[j], x.x, a.x);
          a.y = fmaf(g[j], x.y, a.y);
          a.z = fmaf(g[j], x.z, a.z);
          a.w = fmaf(g[j], x.w, a.w);
        }
      }
      __stcs(reinterpret_cast<float4*>(o), a);
    }
  }
}

// 8 NF3 codes in the low 24 bits of x -> prmt selectors with one code per
// nibble (bit 3 of every nibble clear): codes 0-3 in sel_lo, 4-7 in sel_hi.
__device__ __forceinline__ void nf3_selectors(uint32_t x, uint32_t& sel_lo, uint32_t& sel_hi) {
  const uint32_t y = (x & 0x0000ffffu) | ((x << 4) & 0xffff0000u);  // codes 4-7 -> bits 16..27
  const uint32_t z = (y & 0x00ff00ffu) | ((y << 2) & 0xff00ff00u);  // pairs -> bytes
  const uint32_t w = (z & 0x07070707u) | ((z << 1) & 0x70707070u);  // one code per nibble
  sel_lo = w;
  sel_hi = w >> 16;
}

// Adds a * level[c_i] to acc[0..3] for the 4 codes of nibble selector `sel`.
__device__ __forceinline__ void nf3_fma4(uint32_t sel, float a, float* acc) {
  const uint32_t lo = prmt(kLoBytes0, kLoBytes1, sel);
  const uint32_t hi = prmt(kHiBytes0, kHiBytes1, sel);
  const uint32_t h01 = prmt(lo, hi, 0x5140u);
  const uint32_t h23 = prmt(lo, hi, 0x7362u);
  const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  acc[0] = fmaf(a, f01.x, acc[0]);
  acc[1] = fmaf(a, f01.y, acc[1]);
  acc[2] = fmaf(a, f23.x, acc[2]);
  acc[3] = fmaf(a, f23.y, acc[3]);
}

// Gather + combine of one tile from an NF3 table: unit = (token, 32-element
// half block); the half block's codes are 12 bytes (3 words) per expert row.
template <int NT, bool kExactN>
__device__ __forceinline__ void combine_tile_nf3(const Smem& s, const UnitMap& um,
                                                 const uint8_t* __restrict__ codes,
                                                 const uint16_t* __restrict__ scales, int64_t V, int N,
                                                 int D, int64_t t0, int rows, float* __restrict__ out,
                                                 unsigned* err) {
  constexpr int NP = 8 * NT;
  constexpr int CH = NP < 8 ? NP : 8;
  const int NB = D >> 6;  // 64-element blocks per row
  const int HB = D >> 5;  // half blocks per row
  for (int r = um.r0; r < rows; r += um.rstep) {
    const int id = s.tok_id[r];
    float g[NP];
    load_gates(s.gates + r * NP, g, NP);
    for (int hb = um.v0; hb < HB; hb += um.vstep) {
      float* o = out + (t0 + r) * (int64_t)D + hb * 32;
      if (id < 0 || (int64_t)id >= V) {
        if (hb == 0) atomicOr(err, kErrIndex);
        store_nan(o, 32);
        continue;
      }
      const int b = hb >> 1, half = hb & 1;
      const int64_t blk0 = (int64_t)id * N * NB + b;  // block of expert 0
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j0 = 0; j0 < NP; j0 += CH) {
        uint32_t w[CH][3];
        float sc[CH];
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const int jj = kExactN ? j0 + j : min(j0 + j, N - 1);
          const int64_t blk = blk0 + (int64_t)jj * NB;
          const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes + blk * 24 + half * 12);
          w[j][0] = __ldg(cw);
          w[j][1] = __ldg(cw + 1);
          w[j][2] = __ldg(cw + 2);
          sc[j] = __half2float(__ushort_as_half(__ldg(scales + blk)));
        }
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          if (kExactN || j0 + j < N) {
            const float a = g[j0 + j] * sc[j];
            const uint32_t x0 = w[j][0];
            const uint32_t x1 = __funnelshift_r(w[j][0], w[j][1], 24);
            const uint32_t x2 = __funnelshift_r(w[j][1], w[j][2], 16);
            const uint32_t x3 = w[j][2] >> 8;
            uint32_t sl, sh;
            nf3_selectors(x0, sl, sh);
            nf3_fma4(sl, a, acc + 0);
            nf3_fma4(sh, a, acc + 4);
            nf3_selectors(x1, sl, sh);
            nf3_fma4(sl, a, acc + 8);
            nf3_fma4(sh, a, acc + 12);
            nf3_selectors(x2, sl, sh);
            nf3_fma4(sl, a, acc + 16);
            nf3_fma4(sh, a, acc + 20);
            nf3_selectors(x3, sl, sh);
            nf3_fma4(sl, a, acc + 24);
            nf3_fma4(sh, a, acc + 28);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        __stcs(reinterpret_cast<float4*>(o + i), make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]));
    }
  }
}

struct CombineArgs {
  const int32_t* ids;
  int64_t T;
  const void* h;
  const void* Wr;
  const void* table;      // bf16 / f32 LUT, or NF3 codes
  const uint16_t* scales; // NF3 only
  int64_t V;
  int N, D, TT;
  int64_t n_tiles;
  float* out;
  unsigned* err;
};

// ---------------------------------------------------------------------------
// Two-kernel path for prefill-sized batches (bf16 inputs; bf16 or NF3 table).
//
// 1. router_gates_kernel: persistent CTAs (Wr^T staged once in shared memory)
//    compute the gates of 16-token tiles on the tensor cores (router_tile) and
//    write each token's N gates into the first N floats of that token's own
//    output row -- memory the caller provides and the second kernel overwrites.
// 2. gather_kernel: per CTA one producer thread streams each token's whole row
//    block (N*D*2 contiguous bytes; for NF3 the code block and the scale
//    block) and its gate vector into a ring of shared-memory slots with
//    cp.async.bulk, completion counted on the slot's mbarrier; consumer warps
//    combine from shared memory (16-byte reads, fp32 FMAs) and store fp32
//    outputs.  Bulk copies keep ring-depth x 64 KB in flight per SM without
//    registers or per-thread request slots, so the gather streams at the DRAM
//    rate, and the router's latency no longer sits inside the gather.
// ---------------------------------------------------------------------------
constexpr int kGatherCons = 16;                           // consumer warps
constexpr int kGatherThreads = (kGatherCons + 1) * 32;    // + producer warp
constexpr int kGatherProducer = kGatherCons;
constexpr int kRingBudget = 200 * 1024;                   // bytes of row slots

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Lane 0 of the warp waits (bounded); the result is broadcast to the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, volatile int* abort, unsigned* err) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    if (!mbar_test(b, parity)) {
      const uint64_t t0 = globaltimer();
      for (;;) {
        if (mbar_test(b, parity)) break;
        if (*abort) { ok = false; break; }
        if (globaltimer() - t0 > kWaitLimitNs) {
          *abort = 1;
          atomicOr(err, kErrTimeout);
          ok = false;
          break;
        }
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Slot layout: [0, row_bytes) table row block, [scales_off, +scale_bytes)
// NF3 scales, [gates_off, +NP*4) the token's gates.
struct GatherLayout {
  int n_slots, slot_bytes, scales_off, gates_off;
};

template <int NT>
__global__ void __launch_bounds__(kThreads, 2) router_gates_kernel(const CombineArgs p) {
  constexpr int NP = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Smem s = carve<true, NP>(smem_raw, p.D);
  stage_wrt<NP, kThreads>(s.wrt, static_cast<const uint16_t*>(p.Wr), p.N, p.D);
  __syncthreads();
  for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
    const int64_t t0 = tile * p.TT;
    const int rows = (int)(p.T - t0 < p.TT ? p.T - t0 : p.TT);
    router_tile<true, NT>(s, p.ids, p.h, p.Wr, t0, rows, p.N, p.D);
    for (int i = threadIdx.x; i < rows * NP; i += kThreads) {
      const int r = i / NP, j = i - r * NP;
      p.out[(t0 + r) * (int64_t)p.D + j] = s.gates[i];
    }
    // s.gates is rewritten only after the next tile's first barrier
  }
}

template <int NT, bool kExactN, int kTable, int kChunks>
__global__ void __launch_bounds__(kGatherThreads, 1) gather_kernel(const CombineArgs p, const GatherLayout L) {
  constexpr int NP = 8 * NT;
  constexpr int JC = NP / kChunks;  // expert rows per chunk (kChunks > 1 only with N == NP)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* ring = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + (size_t)L.n_slots * L.slot_bytes);
  uint64_t* empty = full + L.n_slots;
  int* slot_id = reinterpret_cast<int*>(empty + L.n_slots);
  int* abort_flag = slot_id + L.n_slots;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int q = 0; q < L.n_slots; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kGatherCons);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int* abort = abort_flag;
  const int NB = p.D >> 6;
  // bytes of one chunk of a token's row block (bf16: JC rows of D; NF3: all
  // code rows, then the scale rows at scales_off)
  const uint32_t chunk_bytes = kTable == kTableBf16 ? (uint32_t)JC * (uint32_t)p.D * 2u
                                                    : (uint32_t)p.N * (uint32_t)NB * 24u;
  const uint32_t scale_bytes = kTable == kTableBf16 ? 0u : (uint32_t)p.N * (uint32_t)NB * 2u;
  const uint32_t gate_bytes = NP * 4u;
  // this CTA's tokens: t = blockIdx.x + k * gridDim.x, k = 0, 1, ...
  const int64_t n_mine = p.T > blockIdx.x ? (p.T - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (warp == kGatherProducer) {
    // ---------------- producer ----------------
    int64_t k0 = 0;
    int my_id = lane < n_mine ? __ldg(p.ids + blockIdx.x + (int64_t)lane * gridDim.x) : -1;
    int next_id = 32 + lane < n_mine ? __ldg(p.ids + blockIdx.x + (int64_t)(32 + lane) * gridDim.x) : -1;
    uint32_t q = 0, ph = 0, issued = 0;
    bool ok = true;
    for (int64_t k = 0; ok && k < n_mine; ++k) {
      if (k - k0 == 32) {  // next batch of 32 ids; prefetch the one after
        k0 = k;
        my_id = next_id;
        const int64_t kn = k0 + 32 + lane;
        next_id = kn < n_mine ? __ldg(p.ids + blockIdx.x + kn * gridDim.x) : -1;
      }
      const int id = __shfl_sync(0xffffffffu, my_id, (int)(k - k0));
      const bool valid = id >= 0 && (int64_t)id < p.V;
      const int64_t t = blockIdx.x + k * gridDim.x;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        ok = warp_wait(&empty[q], ph ^ 1u, abort, p.err);
        if (!ok) break;
        if (lane == 0) {
          uint8_t* slot = ring + (size_t)q * L.slot_bytes;
          slot_id[q] = id;
          if (valid) {
            const uint32_t bytes = chunk_bytes + (c == 0 ? gate_bytes : 0u) + scale_bytes;
            mbar_expect_tx(&full[q], bytes);
            if (kTable == kTableBf16) {
              bulk_g2s(slot, static_cast<const uint16_t*>(p.table) + ((int64_t)id * p.N + c * JC) * p.D, chunk_bytes,
                       &full[q]);
            } else {
              bulk_g2s(slot, static_cast<const uint8_t*>(p.table) + (int64_t)id * chunk_bytes, chunk_bytes, &full[q]);
              bulk_g2s(slot + L.scales_off, p.scales + (int64_t)id * p.N * NB, scale_bytes, &full[q]);
            }
            if (c == 0) bulk_g2s(slot + L.gates_off, p.out + t * p.D, gate_bytes, &full[q]);
          } else {
            mbar_arrive(&full[q]);  // nothing to copy: the consumers write a NaN row
          }
        }
        ++issued;
        if (++q == (uint32_t)L.n_slots) {
          q = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0) {  // the last copies must have landed before the CTA exits
      for (uint32_t i = 0; i < issued && i < (uint32_t)L.n_slots; ++i) {
        q = q == 0 ? L.n_slots - 1 : q - 1;
        if (q == (uint32_t)L.n_slots - 1) ph ^= 1u;
        mbar_drain(&full[q], ph);
      }
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    // Tokens are dealt to G groups of gw warps (a token has per_tok units:
    // 4-element (8-byte) vectors of a bf16 row, or 32-element NF3 half
    // blocks).  Every warp waits on every slot and releases it, so slot phases
    // stay in step; only the owning group computes.
    const int per_tok = kTable == kTableBf16 ? (p.D >> 2) : (p.D >> 5);
    const int wpt = (per_tok + 31) >> 5;
    const int G = wpt >= kGatherCons ? 1 : kGatherCons / wpt;
    const int gw = kGatherCons / G;
    const int grp = warp / gw;
    const int lt = threadIdx.x - grp * gw * 32;
    const bool one_unit = kTable == kTableBf16 && per_tok <= gw * 32;
    int gsel = 0;  // == token index % G
    uint32_t q = 0, ph = 0;
    bool ok = true;
    for (int64_t k = 0; ok && k < n_mine; ++k) {
      const bool mine = gsel == grp;
      const int64_t t = blockIdx.x + k * gridDim.x;
      float* orow = p.out + t * p.D;
      if (kTable == kTableBf16 && one_unit) {
        // one 4-wide vector per thread, accumulated across the chunks
        float g[NP];
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        bool valid = false;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          ok = warp_wait(&full[q], ph, abort, p.err);
          if (!ok) break;
          const uint8_t* slot = ring + (size_t)q * L.slot_bytes;
          if (c == 0) {
            const int id = slot_id[q];
            valid = id >= 0 && (int64_t)id < p.V;
            if (mine && valid) load_gates(reinterpret_cast<const float*>(slot + L.gates_off), g, NP);
          }
          if (mine && valid && lt < per_tok) {
            const uint2* src = reinterpret_cast<const uint2*>(slot) + lt;
#pragma unroll
            for (int jj = 0; jj < JC; ++jj) {
              const int j = c * JC + jj;
              if (kExactN || j < p.N) {
                const uint2 x = src[jj * per_tok];
                const float gj = g[j];
                a[0] = fmaf(gj, bf16_lo(x.x), a[0]);
                a[1] = fmaf(gj, bf16_hi(x.x), a[1]);
                a[2] = fmaf(gj, bf16_lo(x.y), a[2]);
                a[3] = fmaf(gj, bf16_hi(x.y), a[3]);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[q]);
          if (++q == (uint32_t)L.n_slots) {
            q = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (mine && lt < per_tok) {
          float* o = orow + lt * 4;
          if (valid) {
            __stcs(reinterpret_cast<float4*>(o), make_float4(a[0], a[1], a[2], a[3]));
          } else {
            if (lt == 0) atomicOr(p.err, kErrIndex);
            store_nan(o, 4);
          }
        }
      } else {
        // several units per thread: the whole token is in one slot (kChunks == 1)
        ok = warp_wait(&full[q], ph, abort, p.err);
        if (!ok) break;
        if (mine) {
          const int id = slot_id[q];
          const bool valid = id >= 0 && (int64_t)id < p.V;
          const uint8_t* slot = ring + (size_t)q * L.slot_bytes;
          float g[NP];
          if (valid) load_gates(reinterpret_cast<const float*>(slot + L.gates_off), g, NP);
          const int units = kTable == kTableBf16 ? (p.D >> 3) : per_tok;  // 8-wide vectors here
          for (int v = lt; v < units; v += gw * 32) {
            if (kTable == kTableBf16) {
              float* o = orow + v * 8;
              if (!valid) {
                if (v == 0) atomicOr(p.err, kErrIndex);
                store_nan(o, 8);
                continue;
              }
              const uint4* src = reinterpret_cast<const uint4*>(slot) + v;
              float a[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) a[i] = 0.f;
#pragma unroll
              for (int j = 0; j < NP; ++j) {
                if (kExactN || j < p.N) {
                  const uint4 x = src[(int64_t)j * units];
                  const float gj = g[j];
                  a[0] = fmaf(gj, bf16_lo(x.x), a[0]);
                  a[1] = fmaf(gj, bf16_hi(x.x), a[1]);
                  a[2] = fmaf(gj, bf16_lo(x.y), a[2]);
                  a[3] = fmaf(gj, bf16_hi(x.y), a[3]);
                  a[4] = fmaf(gj, bf16_lo(x.z), a[4]);
                  a[5] = fmaf(gj, bf16_hi(x.z), a[5]);
                  a[6] = fmaf(gj, bf16_lo(x.w), a[6]);
                  a[7] = fmaf(gj, bf16_hi(x.w), a[7]);
                }
              }
              __stcs(reinterpret_cast<float4*>(o), make_float4(a[0], a[1], a[2], a[3]));
              __stcs(reinterpret_cast<float4*>(o + 4), make_float4(a[4], a[5], a[6], a[7]));
            } else {
              float* o = orow + v * 32;
              if (!valid) {
                if (v == 0) atomicOr(p.err, kErrIndex);
                store_nan(o, 32);
                continue;
              }
              const int blk_in_row = v >> 1, half = v & 1;
              const uint16_t* sc_row = reinterpret_cast<const uint16_t*>(slot + L.scales_off);
              float acc[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
              for (int j = 0; j < NP; ++j) {
                if (kExactN || j < p.N) {
                  const int blk = j * NB + blk_in_row;
                  const uint32_t* cw = reinterpret_cast<const uint32_t*>(slot + blk * 24 + half * 12);
                  const uint32_t w0 = cw[0], w1 = cw[1], w2 = cw[2];
                  const float a = g[j] * __half2float(__ushort_as_half(sc_row[blk]));
                  uint32_t sl, sh;
                  nf3_selectors(w0, sl, sh);
                  nf3_fma4(sl, a, acc + 0);
                  nf3_fma4(sh, a, acc + 4);
                  nf3_selectors(__funnelshift_r(w0, w1, 24), sl, sh);
                  nf3_fma4(sl, a, acc + 8);
                  nf3_fma4(sh, a, acc + 12);
                  nf3_selectors(__funnelshift_r(w1, w2, 16), sl, sh);
                  nf3_fma4(sl, a, acc + 16);
                  nf3_fma4(sh, a, acc + 20);
                  nf3_selectors(w2 >> 8, sl, sh);
                  nf3_fma4(sl, a, acc + 24);
                  nf3_fma4(sh, a, acc + 28);
                }
              }
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                __stcs(reinterpret_cast<float4*>(o + i), make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[q]);
        if (++q == (uint32_t)L.n_slots) {
          q = 0;
          ph ^= 1u;
        }
      }
      if (++gsel == G) gsel = 0;
    }
  }
  __syncthreads();
}

template <bool kBf16Router, int NT, int kTable, bool kExactN>
__global__ void __launch_bounds__(kThreads, 2) combine_kernel(const CombineArgs p) {
  constexpr int NP = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const Smem s = carve<kBf16Router, NP>(smem_raw, p.D);
  if (kBf16Router) {
    stage_wrt<NP, kThreads>(s.wrt, static_cast<const uint16_t*>(p.Wr), p.N, p.D);
    __syncthreads();
  }
  const int per_tok = kTable == kTableBf16 ? (p.D >> 3) : kTable == kTableF32 ? (p.D >> 2) : (p.D >> 5);
  const UnitMap um(per_tok);
  for (int64_t tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
    const int64_t t0 = tile * p.TT;
    const int rows = (int)(p.T - t0 < p.TT ? p.T - t0 : p.TT);
    router_tile<kBf16Router, NT>(s, p.ids, p.h, p.Wr, t0, rows, p.N, p.D);
    if (kTable == kTableBf16)
      combine_tile_bf16<NT, kExactN>(s, um, static_cast<const uint16_t*>(p.table), p.V, p.N, p.D, t0, rows,
                                     p.out, p.err);
    else if (kTable == kTableF32)
      combine_tile_f32<NT, kExactN>(s, um, static_cast<const float*>(p.table), p.V, p.N, p.D, t0, rows,
                                    p.out, p.err);
    else
      combine_tile_nf3<NT, kExactN>(s, um, static_cast<const uint8_t*>(p.table), p.scales, p.V, p.N, p.D,
                                    t0, rows, p.out, p.err);
    // the next tile's router writes part/gates/tok_id only after its own
    // __syncthreads, which every thread reaches after finishing this tile
  }
}

// Tokens per tile: the largest TT in {16, 8, 4, 2, 1} that minimises the
// per-SM token count ceil(ceil(T / TT) / n_sm) * TT.
int choose_tile(int64_t T, int n_sm) {
  int best = 1;
  int64_t best_cost = INT64_MAX;
  for (int tt = kTileMax; tt >= 1; tt >>= 1) {
    const int64_t tiles = (T + tt - 1) / tt;
    const int64_t cost = ((tiles + n_sm - 1) / n_sm) * tt;
    if (cost < best_cost) {
      best_cost = cost;
      best = tt;
    }
  }
  return best;
}

template <bool kBf16Router, int NT, int kTable, bool kExactN>
mole_status launch_one(CombineArgs p, cudaStream_t stream) {
  constexpr int NP = 8 * NT;
  const size_t smem = smem_bytes_for<kBf16Router, NP>(p.D);
  if (smem > 227 * 1024) return MOLE_ERR_UNSUPPORTED;
  auto kern = combine_kernel<kBf16Router, NT, kTable, kExactN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  p.TT = choose_tile(p.T, n_sm);
  p.n_tiles = (p.T + p.TT - 1) / p.TT;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess || occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  const int64_t grid = std::min<int64_t>(p.n_tiles, (int64_t)occ * n_sm);
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

template <int NT, bool kExactN, int kTable, int kChunks>
mole_status launch_two_kernel(CombineArgs p, cudaStream_t stream) {
  constexpr int NP = 8 * NT;
  if (p.D < NP) return MOLE_ERR_UNSUPPORTED;  // gates are parked in the output row
  const int64_t NB = p.D / 64;
  GatherLayout L{};
  int64_t off;
  if (kTable == kTableBf16) {
    off = (int64_t)(NP / kChunks) * p.D * 2;
  } else {
    // both bulk copies need 16-byte aligned sources and sizes
    if (((int64_t)p.N * NB) % 8 != 0) return MOLE_ERR_UNSUPPORTED;
    const int64_t code_bytes = (int64_t)p.N * NB * 24;
    L.scales_off = (int)((code_bytes + 127) / 128 * 128);
    off = L.scales_off + (int64_t)p.N * NB * 2;
  }
  L.gates_off = (int)((off + 15) / 16 * 16);
  L.slot_bytes = (int)((L.gates_off + NP * 4 + 127) / 128 * 128);
  L.n_slots = (int)std::min<int64_t>(16, kRingBudget / L.slot_bytes);
  if (L.n_slots < 2 * kChunks) return MOLE_ERR_UNSUPPORTED;
  const size_t gsmem = (size_t)L.n_slots * L.slot_bytes + (size_t)L.n_slots * 20 + 16;
  const size_t rsmem = smem_bytes_for<true, NP>(p.D);
  if (gsmem > 227 * 1024 || rsmem > 227 * 1024) return MOLE_ERR_UNSUPPORTED;
  auto rkern = router_gates_kernel<NT>;
  auto gkern = gather_kernel<NT, kExactN, kTable, kChunks>;
  if (cudaFuncSetAttribute(rkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem) != cudaSuccess ||
      cudaFuncSetAttribute(gkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) != cudaSuccess)
    return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  p.TT = kTileMax;
  p.n_tiles = (p.T + p.TT - 1) / p.TT;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rkern, kThreads, rsmem) != cudaSuccess || occ < 1)
    return MOLE_ERR_UNSUPPORTED;
  rkern<<<(unsigned)std::min<int64_t>(p.n_tiles, (int64_t)occ * n_sm), kThreads, rsmem, stream>>>(p);
  gkern<<<(unsigned)std::min<int64_t>(p.T, n_sm), kGatherThreads, gsmem, stream>>>(p, L);
  return cuda_status(cudaGetLastError());
}

// Batches of at least kTwoKernelMinT tokens (bf16 inputs, bf16 or NF3 table)
// take the router + gather kernel pair; smaller batches and shapes it does not
// cover take the single fused kernel (MOLE_ERR_UNSUPPORTED tells the caller).
constexpr int64_t kTwoKernelMinT = 1024;

template <int kTable>
mole_status launch_staged(const CombineArgs& p, cudaStream_t stream) {
  if (p.T < kTwoKernelMinT) return MOLE_ERR_UNSUPPORTED;
  // bf16 rows above 40 KB per token (e.g. 16 x 2048) travel as two 8-expert
  // halves, so the ring holds twice as many slots in flight
  if (kTable == kTableBf16 && p.N == 16 && (int64_t)p.N * p.D * 2 > 40 * 1024 && p.D / 4 <= kGatherCons * 32)
    return launch_two_kernel<2, true, kTable, 2>(p, stream);
  if (p.N == 16) return launch_two_kernel<2, true, kTable, 1>(p, stream);
  if (p.N == 8) return launch_two_kernel<1, true, kTable, 1>(p, stream);
  if (p.N < 8) return launch_two_kernel<1, false, kTable, 1>(p, stream);
  if (p.N < 16) return launch_two_kernel<2, false, kTable, 1>(p, stream);
  if (p.N == 32) return launch_two_kernel<4, true, kTable, 1>(p, stream);
  return launch_two_kernel<4, false, kTable, 1>(p, stream);
}

template <bool kBf16Router, int kTable>
mole_status launch_combine(const CombineArgs& p, cudaStream_t stream) {
  if (p.N == 16) return launch_one<kBf16Router, 2, kTable, true>(p, stream);
  if (p.N == 8) return launch_one<kBf16Router, 1, kTable, true>(p, stream);
  if (p.N <= 8) return launch_one<kBf16Router, 1, kTable, false>(p, stream);
  if (p.N <= 16) return launch_one<kBf16Router, 2, kTable, false>(p, stream);
  if (p.N == 32) return launch_one<kBf16Router, 4, kTable, true>(p, stream);
  return launch_one<kBf16Router, 4, kTable, false>(p, stream);
}

}  // namespace

// ---- entry points used by api.cu ------------------------------------------

mole_status combine_dispatch(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                             const void* table, const uint16_t* scales, int64_t V, int N, int D,
                             bool bf16_inputs, int table_kind, float* out, cudaStream_t stream) {
  CombineArgs p{};
  p.ids = ids;
  p.T = T;
  p.h = h;
  p.Wr = Wr;
  p.table = table;
  p.scales = scales;
  p.V = V;
  p.N = N;
  p.D = D;
  p.out = out;
  p.err = error_word();
  if (!p.err) return MOLE_ERR_CUDA;
  if (table_kind == kTableNf3) {
    if (!bf16_inputs) return launch_combine<false, kTableNf3>(p, stream);
    const mole_status st = launch_staged<kTableNf3>(p, stream);
    if (st != MOLE_ERR_UNSUPPORTED) return st;
    return launch_combine<true, kTableNf3>(p, stream);
  }
  if (table_kind == kTableBf16) {
    const mole_status st = launch_staged<kTableBf16>(p, stream);
    if (st != MOLE_ERR_UNSUPPORTED) return st;
    return launch_combine<true, kTableBf16>(p, stream);
  }
  return launch_combine<false, kTableF32>(p, stream);
}

void nf3_tables(uint16_t levels[8], float mid[7]) {
  for (int i = 0; i < 8; ++i) levels[i] = kNf3Levels[i];
  for (int i = 0; i < 7; ++i) mid[i] = kNf3Mid[i];
}

// ---- NF3 quantiser ---------------------------------------------------------
// One thread per 64-element block of one (v, j) row, all in IEEE fp32:
// amax -> fp16 scale (saturating, ties to even) -> correctly rounded x / s ->
// number of midpoints below -> 3-bit code at bits [3e, 3e+3) of the block.
__global__ void __launch_bounds__(256) nf3_quantize_kernel(const uint16_t* __restrict__ lut,
                                                           int64_t n_blocks, uint8_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scales) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= n_blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(lut + blk * 64);
  uint32_t xw[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 v = __ldg(src + i);
    xw[4 * i + 0] = v.x;
    xw[4 * i + 1] = v.y;
    xw[4 * i + 2] = v.z;
    xw[4 * i + 3] = v.w;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(xw[i])), fabsf(bf16_hi(xw[i]))));
  const __half s16 = __float2half_rn(fminf(amax, 65504.f));
  const float sc = __half2float(s16);
  const float mid[7] = {MOLE_NF3_MIDPOINTS};
  uint32_t packed[6] = {0u, 0u, 0u, 0u, 0u, 0u};
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
  uint2* dst = reinterpret_cast<uint2*>(codes + blk * 24);
  dst[0] = make_uint2(packed[0], packed[1]);
  dst[1] = make_uint2(packed[2], packed[3]);
  dst[2] = make_uint2(packed[4], packed[5]);
  scales[blk] = __half_as_ushort(s16);
}

mole_status nf3_quantize_launch(const void* lut, int64_t V, int N, int64_t D, uint8_t* codes,
                                uint16_t* scales, cudaStream_t stream) {
  const int64_t n_blocks = V * N * (D / 64);
  if (n_blocks == 0) return MOLE_OK;
  const int64_t grid = (n_blocks + 255) / 256;
  if (grid > 0x7fffffff) return MOLE_ERR_UNSUPPORTED;
  nf3_quantize_kernel<<<(unsigned)grid, 256, 0, stream>>>(static_cast<const uint16_t*>(lut), n_blocks,
                                                           codes, scales);
  return cuda_status(cudaGetLastError());
}

}  // namespace mole
