// combine_common.cuh -- pieces shared by the combine kernels (combine.cu) and
// the id-grouped combine (grouped.cu): the NF3 level tables and decoder, the
// tensor-core router + softmax, the shared-memory carve-up of a router CTA,
// and the bulk-copy / mbarrier helpers of the gather kernels.
#pragma once

#include <math.h>

#include "common.cuh"
#include "nf3.cuh"

namespace mole {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTileMax = 16;  // rows of the m16n8k16 router MMA

// kTableNf3Fine: the NF3 table with 8-element units instead of 32 (four
// times the threads per token, for batches too small to fill the CTA).
enum TableKind { kTableBf16 = 0, kTableF32 = 1, kTableNf3 = 2, kTableNf3Fine = 3 };


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
// Fast path (N == NP, 16-byte aligned Wr, D % 8 == 0): each thread takes 8
// consecutive rows d0..d0+7 and, per 8-expert slice and 4 rows at a time,
// loads their 16-byte pieces, transposes the 4 x 8 bf16 block in registers
// (byte permutes) and writes 8-byte pieces of 8 rows of wrt.
// Otherwise element by element, loads issued in batches before their stores
// so their latencies overlap.
template <int NP, int kNThreads, bool kFast = true>
__device__ __forceinline__ void stage_wrt(uint16_t* wrt, const uint16_t* __restrict__ wr, int N, int D) {
  const int ldw = D + 8;
  if (kFast && N == NP && (reinterpret_cast<uintptr_t>(wr) & 15u) == 0 && (D & 7) == 0) {
    constexpr int Q = NP / 8;  // 16-byte pieces of a Wr row
    // every CTA reads all of Wr at about the same moment: each starts at a
    // different row so the requests spread over the L2 slices
    const int n_tasks = D >> 3;
    const int rot = (int)((blockIdx.x * 97u) % (unsigned)n_tasks);
    for (int k = threadIdx.x; k < n_tasks; k += kNThreads) {
      const int task = k + rot < n_tasks ? k + rot : k + rot - n_tasks;
      const int d0 = task * 8;
      const uint4* src = reinterpret_cast<const uint4*>(wr) + (size_t)d0 * Q;
#pragma unroll
      for (int q = 0; q < Q; ++q) {    // experts 8q .. 8q+7
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // rows d0 + 4hf .. d0 + 4hf + 3
          uint32_t r[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(src + (4 * hf + i) * Q + q);
            r[i][0] = v.x;
            r[i][1] = v.y;
            r[i][2] = v.z;
            r[i][3] = v.w;
          }
#pragma unroll
          for (int m = 0; m < 4; ++m) {  // expert pair (8q + 2m, 8q + 2m + 1)
            const uint2 lo = make_uint2(__byte_perm(r[0][m], r[1][m], 0x5410), __byte_perm(r[2][m], r[3][m], 0x5410));
            const uint2 hi = make_uint2(__byte_perm(r[0][m], r[1][m], 0x7632), __byte_perm(r[2][m], r[3][m], 0x7632));
            *reinterpret_cast<uint2*>(wrt + (size_t)(8 * q + 2 * m) * ldw + d0 + 4 * hf) = lo;
            *reinterpret_cast<uint2*>(wrt + (size_t)(8 * q + 2 * m + 1) * ldw + d0 + 4 * hf) = hi;
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


// ---- router: z[16, N] = h_tile . Wr on the tensor cores, then softmax ----
//
// The logits of a 16-token tile are an m16n8k16 contraction (bf16 in, fp32
// accumulate) with the D dimension split across the kWarps warps: warp w
// takes k-steps w, w + kWarps, ...  The k-slot order inside a 16-wide step is
// permuted (slots 2c,2c+1 <- d+4c+0,1 and 2c+8,2c+9 <- d+4c+2,3) so each
// lane's A piece is one 8-byte load and its B piece one 8-byte shared-memory
// load; a dot product does not depend on that order.

// A fragments (rows g and g+8 of the tile) of one batch of KB k-steps.
template <int KB>
struct RouterA {
  uint2 a0[KB], a1[KB];
};

// Loads the batch of k-steps kb, kb + kWarps, ... (KB of them) of the tile
// [t0, t0 + rows); rows past the tile and k-steps past D read as zero.
template <int KB>
__device__ __forceinline__ void router_load_a(RouterA<KB>& A, const uint16_t* __restrict__ h, int64_t t0, int rows,
                                              int D, int kb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const bool ok0 = g < rows, ok1 = g + 8 < rows;
  const uint16_t* h0 = h + (t0 + (ok0 ? g : 0)) * (int64_t)D + 4 * c;
  const uint16_t* h1 = h + (t0 + (ok1 ? g + 8 : 0)) * (int64_t)D + 4 * c;
  const int ksteps = D >> 4;
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = kb + i * kWarps;
    const bool in = ks < ksteps;
    A.a0[i] = (in && ok0) ? __ldg(reinterpret_cast<const uint2*>(h0 + (ks << 4))) : make_uint2(0u, 0u);
    A.a1[i] = (in && ok1) ? __ldg(reinterpret_cast<const uint2*>(h1 + (ks << 4))) : make_uint2(0u, 0u);
  }
}

// acc += the batch's MMAs against Wr^T staged in shared memory ([NP][D + 8]).
template <int NT, int KB>
__device__ __forceinline__ void router_mma(float (&acc)[NT][4], const RouterA<KB>& A, const uint16_t* wrt, int D,
                                           int kb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3, ldw = D + 8;
  const uint16_t* w = wrt + g * ldw + 4 * c;
  const int ksteps = D >> 4;
#pragma unroll
  for (int i = 0; i < KB; ++i) {
    const int ks = kb + i * kWarps;
    if (ks < ksteps) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint2 b = *reinterpret_cast<const uint2*>(w + nt * 8 * ldw + (ks << 4));
        mma_16816(acc[nt], A.a0[i].x, A.a1[i].x, A.a0[i].y, A.a1[i].y, b.x, b.y);
      }
    }
  }
}

// Each warp's partial logits -> s.part[warp][row][NP].
template <int NT>
__device__ __forceinline__ void router_store_partials(const Smem& s, const float (&acc)[NT][4]) {
  constexpr int NP = 8 * NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  float* pw = s.part + warp * kTileMax * NP;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    pw[g * NP + nt * 8 + 2 * c] = acc[nt][0];
    pw[g * NP + nt * 8 + 2 * c + 1] = acc[nt][1];
    pw[(g + 8) * NP + nt * 8 + 2 * c] = acc[nt][2];
    pw[(g + 8) * NP + nt * 8 + 2 * c + 1] = acc[nt][3];
  }
}

// fp32 router on CUDA cores (fp32 inputs): one warp per token row, lanes
// split D; row sums -> s.part[row][NP].
template <int NT>
__device__ __forceinline__ void router_f32_partials(const Smem& s, const float* __restrict__ h,
                                                    const float* __restrict__ Wr, int64_t t0, int rows, int N,
                                                    int D) {
  constexpr int NP = 8 * NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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

// The whole CTA's barrier (the router's default).
struct CtaSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// Barrier, sum of the partial logits, max-subtracted softmax over the N
// experts (NP lanes per token row; padded experts get gate 0), barrier.  If
// `ids` is given, s.tok_id[r] = ids[t0 + r] is loaded between the barriers
// (before the first one, threads may still be reading the previous tile's
// ids); with kOwnId, thread r stores its argument own_id there instead.  On
// return s.gates[r][j] is valid for r < rows.  The barriers are Sync's (the
// kThreads threads that run the router).
template <bool kBf16Router, int NT, class Sync = CtaSync, bool kOwnId = false>
__device__ __forceinline__ void router_softmax(const Smem& s, int rows, int N, const int32_t* __restrict__ ids,
                                               int64_t t0, int own_id = 0) {
  constexpr int NP = 8 * NT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Sync{}();
  if (kOwnId) {
    if (tid < rows) s.tok_id[tid] = own_id;
  } else if (ids != nullptr && tid < rows) {
    s.tok_id[tid] = __ldg(ids + t0 + tid);
  }
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
  Sync{}();
}

// Persistent router loop over this CTA's 16-token tiles (blockIdx.x,
// blockIdx.x + gridDim.x, ...) for bf16 inputs: Wr^T is staged once, then
// the first batch of A fragments of the next tile is loaded right after the
// current tile's MMAs (into the registers those MMAs just consumed), so the
// loads are in flight during the partial-sum exchange, the softmax and the
// gate stores.  After each tile, sink(t0, rows) reads s.gates.
template <int NT, class Sink>
__device__ __forceinline__ void router_tiles(const Smem& s, const uint16_t* __restrict__ h,
                                             const uint16_t* __restrict__ Wr, int64_t T, int N, int D, Sink&& sink) {
  constexpr int NP = 8 * NT;
  constexpr int KB = 16;
  const int warp = threadIdx.x >> 5;
  const int ksteps = D >> 4;
  const int64_t n_tiles = (T + kTileMax - 1) / kTileMax;
  auto rows_of = [T](int64_t tile) {
    const int64_t t0 = tile * kTileMax;
    return (int)(T - t0 < kTileMax ? T - t0 : kTileMax);
  };
  // under a programmatic dependent launch: let the next kernel get scheduled,
  // then wait for the previous one (it may have produced h, Wr or whatever
  // the sink overwrites)
  pdl_trigger();
  pdl_wait();
  stage_wrt<NP, kThreads>(s.wrt, Wr, N, D);  // before the A registers are live
  RouterA<KB> A;
  int64_t tile = blockIdx.x;
  if (tile < n_tiles) router_load_a<KB>(A, h, tile * kTileMax, rows_of(tile), D, warp);
  __syncthreads();
  for (; tile < n_tiles; tile += gridDim.x) {
    const int64_t t0 = tile * kTileMax;
    const int rows = rows_of(tile);
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    for (int kb = warp; kb < ksteps; kb += kWarps * KB) {
      if (kb != warp) router_load_a<KB>(A, h, t0, rows, D, kb);
      router_mma<NT, KB>(acc, A, s.wrt, D, kb);
    }
    const int64_t next = tile + gridDim.x;
    if (next < n_tiles) router_load_a<KB>(A, h, next * kTileMax, rows_of(next), D, warp);
    router_store_partials<NT>(s, acc);
    router_softmax<true, NT>(s, rows, N, nullptr, t0);
    sink(t0, rows);
    // s.gates is rewritten only after the next tile's first barrier
  }
}

// Router + softmax for one tile of `rows` tokens starting at t0, loads and
// MMAs in batches of 16 k-steps.  On return s.gates[r][j] and s.tok_id[r]
// are valid for r < rows.
template <bool kBf16Router, int NT>
__device__ __forceinline__ void router_tile(const Smem& s, const int32_t* __restrict__ ids,
                                            const void* __restrict__ h_, const void* __restrict__ Wr_,
                                            int64_t t0, int rows, int N, int D) {
  if (kBf16Router) {
    constexpr int KB = 16;
    const uint16_t* h = static_cast<const uint16_t*>(h_);
    const int warp = threadIdx.x >> 5;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    RouterA<KB> A;
    for (int kb = warp; kb < (D >> 4); kb += kWarps * KB) {
      router_load_a<KB>(A, h, t0, rows, D, kb);
      router_mma<NT, KB>(acc, A, s.wrt, D, kb);
    }
    router_store_partials<NT>(s, acc);
  } else {
    router_f32_partials<NT>(s, static_cast<const float*>(h_), static_cast<const float*>(Wr_), t0, rows, N, D);
  }
  router_softmax<kBf16Router, NT>(s, rows, N, ids, t0);
}

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
        if (mbar_test_sleep(b, parity, kSuspendHintNs)) break;
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


}  // namespace
}  // namespace mole
