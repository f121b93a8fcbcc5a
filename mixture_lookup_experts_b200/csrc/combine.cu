// combine.cu -- router + softmax + direct-addressed gather + gate-weighted sum
// over the lookup table (MoLE page, 训练阶段 and 推理阶段: the router sees the
// previous layer's hidden state, every routed expert is active, and each
// token's expert outputs are fetched from the table by its token id).
//
//   out[t, :] = sum_j softmax(h[t] . Wr)_j  LUT[ids[t], j, :]
//
// Two paths:
//  * combine_kernel (small batches, fp32 inputs): one persistent CTA (256
//    threads) walks token tiles of up to 16 tokens: tensor-core router and
//    softmax for the tile (combine_common.cuh), then each thread owns one
//    vector of D of one token and issues the N row loads LUT[id, j, vec] back
//    to back before the fp32 FMAs.
//  * router_gates_kernel + gather_kernel (batches of 1024+ tokens, bf16
//    inputs): the router runs as its own kernel and parks the gates in the
//    output rows; the gather kernel streams whole row blocks into a shared-
//    memory ring with bulk copies and combines from there.
#include "combine_common.cuh"

namespace mole {
namespace {

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

// The same with units of 8 elements (one 24-bit code group of one 64-element
// block per expert row): per element the same FMAs in the same order, so the
// output is bit-identical; four times as many units per token, for tiles
// whose 32-element units would leave most of the CTA's threads idle.
template <int NT, bool kExactN>
__device__ __forceinline__ void combine_tile_nf3_fine(const Smem& s, const UnitMap& um,
                                                      const uint8_t* __restrict__ codes,
                                                      const uint16_t* __restrict__ scales, int64_t V, int N,
                                                      int D, int64_t t0, int rows, float* __restrict__ out,
                                                      unsigned* err) {
  constexpr int NP = 8 * NT;
  const int NB = D >> 6;  // 64-element blocks per row
  const int QB = D >> 3;  // 8-element units per row
  for (int r = um.r0; r < rows; r += um.rstep) {
    const int id = s.tok_id[r];
    float g[NP];
    load_gates(s.gates + r * NP, g, NP);
    for (int u = um.v0; u < QB; u += um.vstep) {
      float* o = out + (t0 + r) * (int64_t)D + u * 8;
      if (id < 0 || (int64_t)id >= V) {
        if (u == 0) atomicOr(err, kErrIndex);
        store_nan(o, 8);
        continue;
      }
      const int b = u >> 3, bit = 24 * (u & 7), wi = bit >> 5, sh = bit & 31;
      const int64_t blk0 = (int64_t)id * N * NB + b;  // block of expert 0
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      uint32_t x[NP];
      float sc[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) {  // every load first, then the arithmetic
        const int jj = kExactN ? j : min(j, N - 1);
        const int64_t blk = blk0 + (int64_t)jj * NB;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes + blk * 24);
        const uint32_t lo = __ldg(cw + wi), hi = wi < 5 ? __ldg(cw + wi + 1) : 0u;
        x[j] = __funnelshift_r(lo, hi, sh) & 0xffffffu;
        sc[j] = __half2float(__ushort_as_half(__ldg(scales + blk)));
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        if (kExactN || j < N) {
          const float a = g[j] * sc[j];
          uint32_t sl, shi;
          nf3_selectors(x[j], sl, shi);
          nf3_fma4(sl, a, acc + 0);
          nf3_fma4(shi, a, acc + 4);
        }
      }
      __stcs(reinterpret_cast<float4*>(o), make_float4(acc[0], acc[1], acc[2], acc[3]));
      __stcs(reinterpret_cast<float4*>(o + 4), make_float4(acc[4], acc[5], acc[6], acc[7]));
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
  router_tiles<NT>(s, static_cast<const uint16_t*>(p.h), static_cast<const uint16_t*>(p.Wr), p.T, p.N, p.D,
                   [&](int64_t t0, int rows) {
                     for (int i = threadIdx.x; i < rows * NP; i += kThreads) {
                       const int r = i / NP, j = i - r * NP;
                       p.out[(t0 + r) * (int64_t)p.D + j] = s.gates[i];
                     }
                   });
}

template <int NT, bool kExactN, int kTable, int kChunks>
__global__ void __launch_bounds__(kGatherThreads, 1) gather_kernel(const CombineArgs p, const GatherLayout L) {
  constexpr int NP = 8 * NT;
  constexpr int JC = NP / kChunks;  // expert rows per chunk
  static_assert(kChunks == 1 || kExactN, "split row blocks need N == NP");
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
  pdl_trigger();
  pdl_wait();  // the router's gates are complete
  volatile int* abort = abort_flag;
  const int NB = p.D >> 6;
  // bytes of one chunk of a token's row block (bf16: JC rows of D; NF3: all
  // code rows, then the scale rows at scales_off)
  // (with a padded expert count only the N real rows are copied: the rows
  // after them belong to the next id, or lie past the table's end)
  const uint32_t chunk_bytes = kTable == kTableBf16 ? (uint32_t)(kExactN ? JC : p.N) * (uint32_t)p.D * 2u
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
  // launched with programmatic stream serialization: the launch overlaps the
  // previous kernel's tail; every input is read after it has completed
  pdl_trigger();
  pdl_wait();
  if (kBf16Router) {
    // (the element-wise staging: the fused kernel's registers are spoken for)
    stage_wrt<NP, kThreads, false>(s.wrt, static_cast<const uint16_t*>(p.Wr), p.N, p.D);
    __syncthreads();
  }
  const int per_tok = kTable == kTableBf16 ? (p.D >> 3)
                      : kTable == kTableF32 ? (p.D >> 2)
                      : kTable == kTableNf3Fine ? (p.D >> 3)
                                                : (p.D >> 5);
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
    else if (kTable == kTableNf3Fine)
      combine_tile_nf3_fine<NT, kExactN>(s, um, static_cast<const uint8_t*>(p.table), p.scales, p.V, p.N, p.D,
                                         t0, rows, p.out, p.err);
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
  return cuda_status(launch_pdl(kern, (unsigned)grid, kThreads, smem, stream, p));
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
  // the tensor-core router for NF3 tables only: the bf16 paths (this one,
  // the grouped kernels) all take the mma.sync router arithmetic
  if (kTable != kTableBf16 && router_tc_supported(p.T, p.N, p.D, p.h, p.Wr)) {
    const mole_status st = router_tc_launch(p.h, p.Wr, p.T, p.D, false, p.out, nullptr, nullptr, stream);
    if (st != MOLE_OK) return st;
  } else if (launch_pdl(rkern, (unsigned)std::min<int64_t>(p.n_tiles, (int64_t)occ * n_sm), kThreads, rsmem, stream,
                        p) != cudaSuccess) {
    return MOLE_ERR_CUDA;
  }
  if (launch_pdl(gkern, (unsigned)std::min<int64_t>(p.T, n_sm), kGatherThreads, gsmem, stream, p, L) != cudaSuccess)
    return MOLE_ERR_CUDA;
  return MOLE_OK;
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
    // 8-element units where 32-element ones would leave threads idle
    const int n_sm = num_sms();
    if (n_sm > 0 && T * (int64_t)(D >> 5) < (int64_t)n_sm * kThreads) return launch_combine<true, kTableNf3Fine>(p, stream);
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
// One thread per 64-element block of one (v, j) row, the quantiser of
// nf3.cuh in two passes over the block's 128 bytes (the second from L1) so
// that no thread holds the whole block in registers and 4 CTAs fit per SM:
// amax -> fp16 scale (saturating, ties to even); then per element the number
// of midpoints below the correctly rounded x / s, found by comparing x with
// the block's 7 thresholds on the bf16 grid (packed compares of bf16 pairs)
// -> 3-bit code at bits [3e, 3e+3).
__global__ void __launch_bounds__(256, 4) nf3_quantize_kernel(const uint16_t* __restrict__ lut,
                                                              int64_t n_blocks, uint8_t* __restrict__ codes,
                                                              uint16_t* __restrict__ scales) {
  const int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (blk >= n_blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(lut + blk * 64);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[q])), fabsf(bf16_hi(w[q]))));
  }
  const __half s16 = nf3_scale(amax);
  const float sc = __half2float(s16);
  uint32_t packed[6] = {0u, 0u, 0u, 0u, 0u, 0u};
  if (sc == 0.f) {
#pragma unroll
    for (int e = 0; e < 64; ++e) nf3_put(packed, e, (uint32_t)kNf3ZeroCode);
  } else {
    float t[7];
    nf3_thresholds(sc, t);
    __nv_bfloat162 t2[7];
    nf3_threshold_pairs(t, t2);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t c = nf3_code_pair(w[q], t2);
        nf3_put(packed, 8 * i + 2 * q, c & 0xffffu);
        nf3_put(packed, 8 * i + 2 * q + 1, c >> 16);
      }
    }
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
