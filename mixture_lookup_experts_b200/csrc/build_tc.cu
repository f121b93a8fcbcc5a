// build_tc.cu -- table build on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA).  MoLE page, 推理阶段: the embedding matrix is fed to
// every routed expert, LUT[v, j, :] = act(E[v] . W1[j]) . W2[j].
//
// The build is two batched bf16 GEMMs per group of experts (fp32 accumulate):
//   GEMM1  H[e]          = act(E . W1[e])   E [V, D] K-major, W1[e] [D, Dr] N-major
//   GEMM2  LUT[:, e, :]  = H[e] . W2[e]     H[e] [V, Dr] K-major, W2[e] [Dr, D] N-major
// H is rounded to bf16 (the operand type of the second contraction).
//
// The same kernels serve the training backward, whose GEMMs take transposed
// operands: A may also be MN-major (A[m, k] with m contiguous, loaded as
// 64(M) x 64(K) boxes) and B K-major (B[k, n] with k contiguous, loaded as
// 64(K) x 128(N) boxes); an operand's expert coordinate may also step its
// innermost coordinate (a matrix of rows of N experts' blocks); the
// contraction may run over several experts' K ranges (a sum over experts);
// the epilogue may scale by the activation's derivative (bf16 out), or add
// into an fp32 output, optionally through a row map.
//
// Kernel: persistent, one CTA per SM, 10 warps with fixed roles
//   warp 0      TMA producer (one lane): A box 64(K) x 128(M), B four boxes
//               64(N) x 64(K), all 128-byte swizzled, into a 4-stage ring;
//   warp 1      TMEM owner + MMA issuer (one lane): tcgen05.mma kind::f16,
//               M=128 N=256 K=16, accumulators double-buffered in TMEM
//               (2 x 256 fp32 columns = all 512), tcgen05.commit frees smem
//               stages and signals a finished accumulator;
//   warps 2..9  epilogue, two warps per TMEM lane quadrant (each takes half of
//               the 256 columns): tcgen05.ld 32 lanes x 32 columns, activation,
//               bf16 rounding, 16-byte stores (row stride ldc, so the second
//               GEMM writes the strided LUT[:, e, :] directly).
// Tiles (expert, m-block, n-block) are dealt round-robin to the CTAs with the
// n-block fastest, so concurrently running CTAs share the A rows and the whole
// B[e] panel through L2.
//
// Every wait is bounded (a few seconds of %globaltimer); a wait that runs out
// sets the device error word, all roles leave their loops, outstanding copies
// and MMAs are drained with bounded waits, and TMEM is released before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "nf3.cuh"

namespace mole {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB
constexpr int B_BOX = BK * 64 * 2;    // 8 KB: 64 k-rows of 64 n
constexpr int B_STAGE = BK * BN * 2;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;  // 512: two accumulators
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kSmemBytes = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 256 /*barriers*/;

// Instruction descriptor, kind::f16: D fp32 (bits 4-5), A and B bf16 (bits
// 7-9, 10-12), A MN-major (bit 15) or K-major, B MN-major (bit 16) or
// K-major, N/8 at bits 17-22, M/16 at bits 24-28.
template <bool kAmn, bool kBk, int kM>
constexpr uint32_t idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (kAmn ? 1u << 15 : 0u) | (kBk ? 0u : 1u << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}
constexpr int A_BOX = 64 * BK * 2;  // 8 KB: an MN-major A box, 64(M) x 64(K)
constexpr int BK_BOX = BK * 128 * 2;  // 16 KB: a K-major B box, 64(K) x 128(N)

struct Params {
  int M, N, K;            // per expert: C[M, N] = act(A[M, K] . B[K, N])
  // TMA coordinates of expert e's operand: (x + e * X_e0, y, e * X_e2), x
  // the operand's innermost coordinate (A: a_e2 = 0 shares A by all experts)
  int a_e0, a_e2, b_e0, b_e2;
  // > 0: the contraction of output "expert" s runs over the K ranges of the
  // k_experts experts s * k_experts .. s * k_experts + k_experts - 1 (a sum
  // over experts), expert c's operands at coordinates as above with e = c
  int k_experts;
  int act;
  uint16_t* C;            // bf16 output
  int64_t ldc;            // elements between rows of C
  int64_t c_estride;      // elements between experts of C
  int m_blocks, n_blocks;
  int64_t tiles;
  unsigned* err;
  // fp32 output instead: Cf[e][r, n] = acc + add0[e][r, n] + add1[e][r, n]
  // (either term may be absent), all three row-major with stride ldc and
  // cf_estride elements between experts, r = c_rowmap[m] (or m if absent);
  // Cf may be add0 or add1 (each element is read, then written, by one thread)
  float* Cf;
  const float* add0;
  const float* add1;
  int64_t cf_estride;
  const int* c_rowmap;
  // bf16 output scaled by the activation's derivative instead (training
  // backward): C = bf16(acc * act'(grad_pre[e][m, n])), grad_pre fp32 with
  // stride ldc and pre_estride elements between experts
  const float* grad_pre;
  // NF3 table instead (second build GEMM): the bf16-rounded outputs of each
  // 64-column block quantised in registers; block (m, e, b) at
  // codes + (m * q_row + e * q_e + b) * 24 and scales + the same index
  uint8_t* codes;
  uint16_t* scales;
  int64_t q_row, q_e;
  // also the fp32 pre-activation of the bf16 output (training): element
  // (e, m, n) at pre + e * pre_estride + m * ldc + n
  float* pre;
  int64_t pre_estride;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 layout version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc_v,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc_v), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptors of k-step k (16 elements of K) of a stage:
// K-major operands advance 32 bytes inside the 128-byte swizzle atom (8-row
// groups 1024 bytes apart); MN-major ones advance 16 rows of 128 bytes
// (2048 bytes), their 64-element MN groups one box apart.
template <bool kKMajor>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k, uint32_t mn_group_bytes) {
  if constexpr (kKMajor) return sw128_desc(base + 32 * k, 16, 1024);
  else return sw128_desc(base + 2048 * k, mn_group_bytes, 1024);
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Activation, bf16 rounding and 16-byte stores of one 32-column chunk of a
// row held in registers (the activation is a template argument so the
// per-element loop has no branch).
template <int ACT>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], uint16_t* dst_row) {
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float x0 = act_t<ACT>(__uint_as_float(r[2 * i]));
    const float x1 = act_t<ACT>(__uint_as_float(r[2 * i + 1]));
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
    packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  uint4* dst = reinterpret_cast<uint4*>(dst_row);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

__device__ __forceinline__ void store_chunk_act(int act, const uint32_t (&r)[32], uint16_t* dst_row) {
  switch (act) {
    case MOLE_ACT_GELU_ERF: store_chunk<MOLE_ACT_GELU_ERF>(r, dst_row); break;
    case MOLE_ACT_GELU_TANH: store_chunk<MOLE_ACT_GELU_TANH>(r, dst_row); break;
    case MOLE_ACT_RELU: store_chunk<MOLE_ACT_RELU>(r, dst_row); break;
    case MOLE_ACT_SILU: store_chunk<MOLE_ACT_SILU>(r, dst_row); break;
    default: store_chunk<MOLE_ACT_IDENTITY>(r, dst_row); break;
  }
}

// The fp32 epilogue: 32 columns of one row, plus up to two fp32 terms, at
// element offset `off` of Cf, add0 and add1.
__device__ __forceinline__ void store_chunk_f32(const uint32_t (&r)[32], const Params& p, int64_t off) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (p.add0 != nullptr) {
    const float4* a = reinterpret_cast<const float4*>(p.add0 + off);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 t = a[q];
      v[4 * q] += t.x;
      v[4 * q + 1] += t.y;
      v[4 * q + 2] += t.z;
      v[4 * q + 3] += t.w;
    }
  }
  if (p.add1 != nullptr) {
    const float4* a = reinterpret_cast<const float4*>(p.add1 + off);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 t = a[q];
      v[4 * q] += t.x;
      v[4 * q + 1] += t.y;
      v[4 * q + 2] += t.z;
      v[4 * q + 3] += t.w;
    }
  }
  float4* o = reinterpret_cast<float4*>(p.Cf + off);
#pragma unroll
  for (int q = 0; q < 8; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// The derivative epilogue: 32 columns of one row times act'(pre), rounded to
// bf16, 16-byte stores.
template <int ACT>
__device__ __forceinline__ void store_chunk_grad(const uint32_t (&r)[32], const float* pre, uint16_t* dst_row) {
  const float4* pv = reinterpret_cast<const float4*>(pre);
  uint32_t packed[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 u = pv[q];
    const __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float(r[4 * q]) * act_grad_t<ACT>(u.x),
                                                    __uint_as_float(r[4 * q + 1]) * act_grad_t<ACT>(u.y));
    const __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float(r[4 * q + 2]) * act_grad_t<ACT>(u.z),
                                                    __uint_as_float(r[4 * q + 3]) * act_grad_t<ACT>(u.w));
    packed[2 * q] = *reinterpret_cast<const uint32_t*>(&lo);
    packed[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&hi);
  }
  uint4* dst = reinterpret_cast<uint4*>(dst_row);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
}

__device__ __forceinline__ void store_chunk_grad_act(int act, const uint32_t (&r)[32], const float* pre,
                                                     uint16_t* dst_row) {
  switch (act) {
    case MOLE_ACT_GELU_ERF: store_chunk_grad<MOLE_ACT_GELU_ERF>(r, pre, dst_row); break;
    case MOLE_ACT_GELU_TANH: store_chunk_grad<MOLE_ACT_GELU_TANH>(r, pre, dst_row); break;
    case MOLE_ACT_RELU: store_chunk_grad<MOLE_ACT_RELU>(r, pre, dst_row); break;
    case MOLE_ACT_SILU: store_chunk_grad<MOLE_ACT_SILU>(r, pre, dst_row); break;
    default: store_chunk_grad<MOLE_ACT_IDENTITY>(r, pre, dst_row); break;
  }
}

// The NF3 epilogue: two 32-column chunks (one 64-element block) of one row,
// rounded to bf16 as the table would hold them, quantised, codes and scale
// stored.
__device__ __forceinline__ void store_block_nf3(const uint32_t (&r0)[32], const uint32_t (&r1)[32], const Params& p,
                                                int64_t blk) {
  uint32_t xw[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
    const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
    xw[i] = *reinterpret_cast<const uint32_t*>(&a);
    xw[16 + i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  uint32_t packed[6];
  const uint16_t s16 = nf3_quantize_block(xw, packed);
  uint2* dst = reinterpret_cast<uint2*>(p.codes + blk * 24);
  dst[0] = make_uint2(packed[0], packed[1]);
  dst[1] = make_uint2(packed[2], packed[3]);
  dst[2] = make_uint2(packed[4], packed[5]);
  p.scales[blk] = s16;
}

// One epilogue warp's columns of one tile: BN/64 chunks of 32 from chunk0.
__device__ __forceinline__ void epilogue_tile(const Params& p, uint32_t taddr, int e, int m, int nb, int chunk0,
                                              uint16_t* crow) {
  if (p.codes != nullptr) {
    for (int chunk = chunk0; chunk < chunk0 + BN / 64; chunk += 2) {
      const int col0 = nb * BN + chunk * 32;
      if (col0 >= p.N) break;  // warp-uniform; p.N % 64 == 0
      uint32_t r0[32], r1[32];
      tmem_ld32(taddr + chunk * 32, r0);
      tmem_ld32(taddr + (chunk + 1) * 32, r1);
      if (m < p.M) store_block_nf3(r0, r1, p, (int64_t)m * p.q_row + (int64_t)e * p.q_e + col0 / 64);
    }
    return;
  }
  for (int chunk = chunk0; chunk < chunk0 + BN / 64; ++chunk) {
    const int col0 = nb * BN + chunk * 32;
    if (col0 >= p.N) break;  // warp-uniform
    uint32_t r[32];
    tmem_ld32(taddr + chunk * 32, r);
    if (m < p.M) {
      if (p.Cf != nullptr) {
        const int64_t row = p.c_rowmap != nullptr ? (int64_t)p.c_rowmap[m] : (int64_t)m;
        store_chunk_f32(r, p, (int64_t)e * p.cf_estride + row * p.ldc + col0);
      } else if (p.grad_pre != nullptr) {
        store_chunk_grad_act(p.act, r, p.grad_pre + (int64_t)e * p.pre_estride + (int64_t)m * p.ldc + col0,
                             crow + col0);
      } else {
        if (p.pre != nullptr) {
          float4* dst = reinterpret_cast<float4*>(p.pre + (int64_t)e * p.pre_estride + (int64_t)m * p.ldc + col0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                 __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        }
        store_chunk_act(p.act, r, crow + col0);
      }
    }
  }
}

__device__ __forceinline__ void decode_tile(const Params& p, int64_t tile, int& e, int& mb, int& nb) {
  const int64_t per_e = (int64_t)p.m_blocks * p.n_blocks;
  e = (int)(tile / per_e);
  const int64_t r = tile - (int64_t)e * per_e;
  mb = (int)(r / p.n_blocks);
  nb = (int)(r - (int64_t)mb * p.n_blocks);
}

// Expert coordinate and k-block of step `kbt` of a tile of output expert e.
__device__ __forceinline__ void k_step(const Params& p, int e, int kbt, int kblocks, int& ec, int& kb) {
  if (p.k_experts > 0) {
    const int q = kbt / kblocks;
    ec = e * p.k_experts + q;
    kb = kbt - q * kblocks;
  } else {
    ec = e;
    kb = kbt;
  }
}

// TMA loads of one stage (single CTA): A rows m0.., B columns n0.. (BN).
template <bool kAmn, bool kBk>
__device__ __forceinline__ void load_stage(uint8_t* sa, uint8_t* sb, const CUtensorMap* ma, const CUtensorMap* mb,
                                           uint64_t* bar, const Params& p, int ec, int kb, int m0, int n0) {
  const int k0 = kb * BK;
  if constexpr (kAmn) {
#pragma unroll
    for (int q = 0; q < BM / 64; ++q) tma_load_3d(sa + q * A_BOX, ma, bar, m0 + q * 64 + ec * p.a_e0, k0, ec * p.a_e2);
  } else {
    tma_load_3d(sa, ma, bar, k0 + ec * p.a_e0, m0, ec * p.a_e2);
  }
  if constexpr (kBk) {
#pragma unroll
    for (int q = 0; q < BN / 128; ++q)
      tma_load_3d(sb + q * BK_BOX, mb, bar, k0 + ec * p.b_e0, n0 + q * 128, ec * p.b_e2);
  } else {
#pragma unroll
    for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * B_BOX, mb, bar, n0 + q * 64 + ec * p.b_e0, k0, ec * p.b_e2);
  }
}

template <bool kAmn, bool kBk>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = (p.K + BK - 1) / BK;
  const int ksteps = kblocks * (p.k_experts > 0 ? p.k_experts : 1);
  constexpr uint32_t kId = idesc<kAmn, kBk, BM>();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
        int e, mb, nb;
        decode_tile(p, tile, e, mb, nb);
        for (int kbt = 0; kbt < ksteps; ++kbt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort, p.err)) {
            ok = false;
            break;
          }
          int ec, kb;
          k_step(p, e, kbt, kblocks, ec, kb);
          mbar_expect_tx(&full[s], STAGE_BYTES);
          load_stage<kAmn, kBk>(sA + s * A_STAGE, sB + s * B_STAGE, &map_a, &map_b, &full[s], p, ec, kb, mb * BM,
                                nb * BN);
        }
      }
      // Drain: the last (up to STAGES) issued loads must have landed before exit.
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
      for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % STAGES], (i / STAGES) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t it = 0, tl = 0;
      bool ok = true, issued = false;
      for (int64_t tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x, ++tl) {
        const uint32_t acc = tl & 1u, aph = (tl >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        for (int kbt = 0; kbt < ksteps; ++kbt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * A_STAGE), b0 = smem_u32(sB + s * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma(d_tmem, operand_desc<!kAmn>(a0, k, A_BOX), operand_desc<kBk>(b0, k, B_BOX), kId, (kbt | k) != 0);
          issued = true;
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      if (!ok && issued) {
        // Make sure no MMA still writes TMEM when it is released.
        umma_commit(drain);
        mbar_drain(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int quad = warp & 3;                 // TMEM lanes this warp may access
    const int chunk0 = ((warp - 2) >> 2) * (BN / 64);  // first of its BN/64 column chunks
    uint32_t tl = 0;
    for (int64_t tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++tl) {
      const uint32_t acc = tl & 1u, aph = (tl >> 1) & 1u;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&tfull[acc], aph, abort, p.err);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      int e, mb, nb;
      decode_tile(p, tile, e, mb, nb);
      const int m = mb * BM + quad * 32 + lane;
      uint16_t* crow = p.C + (int64_t)e * p.c_estride + (int64_t)m * p.ldc;
      epilogue_tile(p, tmem_base + ((uint32_t)(quad * 32) << 16) + acc * ACC_COLS, e, m, nb, chunk0, crow);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (tcgen05 cta_group::2): a cluster of 2 CTAs computes a
// 256 x 256 tile.  Each CTA TMA-loads its own 128 rows of A and its own 128
// columns of B (no multicast); the even CTA issues M=256 N=256 K=16 MMAs that
// read both CTAs' shared memory and write each CTA's 128 x 256 fp32
// accumulator into its own TMEM.  Per SM this halves the B bytes per flop, so
// a 6-stage ring of 32 KB per CTA buffers 1.5x more MMA work than the 1-CTA
// ring.  Barriers: full[s] lives in the even CTA (both CTAs' copies complete
// on it); empty[s] and tfull[a] exist in both CTAs and are signalled by one
// multicast tcgen05.commit; tempty[a] lives in the even CTA and counts the
// epilogue warps of both CTAs.
// ---------------------------------------------------------------------------
constexpr int STAGES2 = 6;
constexpr int A_STAGE2 = BM * BK * 2;        // this CTA's 128 rows, 16 KB
constexpr int B_STAGE2 = BK * (BN / 2) * 2;  // this CTA's 128 columns, 16 KB
constexpr int STAGE2_BYTES = A_STAGE2 + B_STAGE2;
constexpr int kSmemBytes2 = 1024 + STAGES2 * STAGE2_BYTES + 256;


__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc_v,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc_v), "r"(accumulate)
      : "memory");
}

// TMA loads of one stage of one CTA of a pair: its 128 rows of A from m0,
// its 128 columns of B from n0; completion on the even CTA's barrier.
template <bool kAmn, bool kBk>
__device__ __forceinline__ void load_stage_pair(uint8_t* sa, uint8_t* sb, const CUtensorMap* ma,
                                                const CUtensorMap* mb, uint32_t bar, const Params& p, int ec, int kb,
                                                int m0, int n0) {
  const int k0 = kb * BK;
  if constexpr (kAmn) {
#pragma unroll
    for (int q = 0; q < BM / 64; ++q)
      tma_load_3d_pair(sa + q * A_BOX, ma, bar, m0 + q * 64 + ec * p.a_e0, k0, ec * p.a_e2);
  } else {
    tma_load_3d_pair(sa, ma, bar, k0 + ec * p.a_e0, m0, ec * p.a_e2);
  }
  if constexpr (kBk) {
    tma_load_3d_pair(sb, mb, bar, k0 + ec * p.b_e0, n0, ec * p.b_e2);
  } else {
#pragma unroll
    for (int q = 0; q < BN / 128; ++q)
      tma_load_3d_pair(sb + q * B_BOX, mb, bar, n0 + q * 64 + ec * p.b_e0, k0, ec * p.b_e2);
  }
}

// Arrive on the barrier at this offset in the CTAs of `mask` when all prior
// MMAs of this thread are complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __noinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (globaltimer() - t0 < ns) {
  }
}

template <bool kAmn, bool kBk>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES2 * A_STAGE2;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES2 * B_STAGE2);
  uint64_t* empty = full + STAGES2;
  uint64_t* tfull = empty + STAGES2;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = (p.K + BK - 1) / BK;
  const int ksteps = kblocks * (p.k_experts > 0 ? p.k_experts : 1);
  constexpr uint32_t kId = idesc<kAmn, kBk, 2 * BM>();
  const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  bool aborted = false;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = pair; ok && tile < p.tiles; tile += n_pairs) {
        int e, mb, nb;
        decode_tile(p, tile, e, mb, nb);
        for (int kbt = 0; kbt < ksteps; ++kbt, ++it) {
          const uint32_t s = it % STAGES2, ph = (it / STAGES2) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort, p.err)) {
            ok = false;
            break;
          }
          int ec, kb;
          k_step(p, e, kbt, kblocks, ec, kb);
          if (leader) mbar_expect_tx(&full[s], 2 * STAGE2_BYTES);
          const uint32_t bar = mapa(smem_u32(&full[s]), 0);
          load_stage_pair<kAmn, kBk>(sA + s * A_STAGE2, sB + s * B_STAGE2, &map_a, &map_b, bar, p, ec, kb,
                                     mb * 2 * BM + (int)rank * BM, nb * BN + (int)rank * (BN / 2));
        }
      }
      if (leader) {
        const uint32_t first = it > (uint32_t)STAGES2 ? it - STAGES2 : 0u;
        for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % STAGES2], (i / STAGES2) & 1u);
      }
      aborted = !ok;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA) ----------------
      uint32_t it = 0, tl = 0;
      bool ok = true, issued = false;
      for (int64_t tile = pair; ok && tile < p.tiles; tile += n_pairs, ++tl) {
        const uint32_t acc = tl & 1u, aph = (tl >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        for (int kbt = 0; kbt < ksteps; ++kbt, ++it) {
          const uint32_t s = it % STAGES2, ph = (it / STAGES2) & 1u;
          if (!mbar_wait(&full[s], ph, abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * A_STAGE2), b0 = smem_u32(sB + s * B_STAGE2);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_pair(d_tmem, operand_desc<!kAmn>(a0, k, A_BOX), operand_desc<kBk>(b0, k, B_BOX), kId,
                      (kbt | k) != 0);
          issued = true;
          umma_commit_pair(&empty[s], 0x3);
        }
        if (ok) umma_commit_pair(&tfull[acc], 0x3);
      }
      if (!ok && issued) {
        umma_commit_pair(drain, 0x1);
        mbar_drain(drain, 0);
      }
      aborted = !ok;
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9 of both CTAs) ----------------
    const int quad = warp & 3;
    const int chunk0 = ((warp - 2) >> 2) * (BN / 64);
    uint32_t tl = 0;
    for (int64_t tile = pair; tile < p.tiles; tile += n_pairs, ++tl) {
      const uint32_t acc = tl & 1u, aph = (tl >> 1) & 1u;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&tfull[acc], aph, abort, p.err);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        aborted = true;
        break;
      }
      tc_fence_after();
      int e, mb, nb;
      decode_tile(p, tile, e, mb, nb);
      const int m = mb * 2 * BM + (int)rank * BM + quad * 32 + lane;
      uint16_t* crow = p.C + (int64_t)e * p.c_estride + (int64_t)m * p.ldc;
      epilogue_tile(p, tmem_base + ((uint32_t)(quad * 32) << 16) + acc * ACC_COLS, e, m, nb, chunk0, crow);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa(smem_u32(&tempty[acc]), 0));
    }
  }

  // A CTA that gave up leaves its peer's copies time to land before the pair
  // passes the final cluster barrier (the even CTA drains its own barriers).
  if (__syncthreads_or(aborted ? 1 : 0) && !leader) spin_ns(10000000ull);
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 tensor map {d0 (contiguous), d1, d2} with a box {64, box1, 1},
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
              uint64_t s2_bytes, uint32_t box1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kAmn, bool kBk>
mole_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, Params p, bool pair_tiles,
                        cudaStream_t stream) {
  static bool attr_set[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOLE_ERR_CUDA;
  if (!attr_set[dev][pair_tiles]) {
    const cudaError_t e = pair_tiles ? cudaFuncSetAttribute(gemm_tc2_kernel<kAmn, kBk>,
                                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes2)
                                     : cudaFuncSetAttribute(gemm_tc_kernel<kAmn, kBk>,
                                                            cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return MOLE_ERR_CUDA;
    attr_set[dev][pair_tiles] = true;
  }
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  if (pair_tiles) {
    const int64_t pairs = std::min<int64_t>(p.tiles, n_sm / 2);
    gemm_tc2_kernel<kAmn, kBk><<<(unsigned)(2 * pairs), kThreads, kSmemBytes2, stream>>>(ma, mb, p);
  } else {
    const int64_t grid = std::min<int64_t>(p.tiles, n_sm);
    gemm_tc_kernel<kAmn, kBk><<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(ma, mb, p);
  }
  return cuda_status(cudaGetLastError());
}

mole_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, Params p, bool pair_tiles,
                        cudaStream_t stream) {
  return launch_gemm<false, false>(ma, mb, p, pair_tiles, stream);
}

}  // namespace

mole_status build_tc_any(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N, int64_t Dr,
                         int act, void* lut, uint8_t* codes, uint16_t* scales, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

bool shared_ffn_tc_supported(int64_t T, int64_t D, int64_t Ds, const void* h, const void* W1s, const void* W2s,
                             const void* add0, const void* add1, const void* out, const void* ws) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return false;
  if (D % 64 != 0 || Ds % 64 != 0 || T < 1 || T > (1LL << 31) - 1 || D > (1LL << 31) - 1 || Ds > (1LL << 31) - 1)
    return false;
  return aligned16(h) && aligned16(W1s) && aligned16(W2s) && aligned16(add0) && aligned16(add1) && aligned16(out) &&
         aligned16(ws) && encode_fn();
}

mole_status shared_ffn_tc(const void* h, const void* W1s, const void* W2s, int64_t T, int64_t D, int64_t Ds, int act,
                          const float* add0, const float* add1, float* out, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  if (ws_bytes < (size_t)T * Ds * 2) return MOLE_ERR_WORKSPACE;
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  uint16_t* H = static_cast<uint16_t*>(ws);
  const bool pair_tiles = T >= 2 * BM;
  const int mtile = pair_tiles ? 2 * BM : BM;
  // GEMM1: H = act(h . W1s), bf16
  CUtensorMap ma, mb;
  if (!make_map(&ma, h, D, T, 1, D * 2, T * D * 2, BM)) return MOLE_ERR_CUDA;
  if (!make_map(&mb, W1s, Ds, D, 1, Ds * 2, D * Ds * 2, BK)) return MOLE_ERR_CUDA;
  Params p1{};
  p1.M = (int)T;
  p1.N = (int)Ds;
  p1.K = (int)D;
  p1.a_e2 = 0;
  p1.b_e2 = 1;
  p1.act = act;
  p1.C = H;
  p1.ldc = Ds;
  p1.c_estride = T * Ds;
  p1.m_blocks = (int)((T + mtile - 1) / mtile);
  p1.n_blocks = (int)((Ds + BN - 1) / BN);
  p1.tiles = (int64_t)p1.m_blocks * p1.n_blocks;
  p1.err = err;
  mole_status st = launch_gemm(ma, mb, p1, pair_tiles, stream);
  if (st != MOLE_OK) return st;
  // GEMM2: out = H . W2s + add0 + add1, fp32
  if (!make_map(&ma, H, Ds, T, 1, Ds * 2, T * Ds * 2, BM)) return MOLE_ERR_CUDA;
  if (!make_map(&mb, W2s, D, Ds, 1, D * 2, Ds * D * 2, BK)) return MOLE_ERR_CUDA;
  Params p2{};
  p2.M = (int)T;
  p2.N = (int)D;
  p2.K = (int)Ds;
  p2.a_e2 = 1;
  p2.b_e2 = 1;
  p2.act = MOLE_ACT_IDENTITY;
  p2.ldc = D;
  p2.m_blocks = (int)((T + mtile - 1) / mtile);
  p2.n_blocks = (int)((D + BN - 1) / BN);
  p2.tiles = (int64_t)p2.m_blocks * p2.n_blocks;
  p2.err = err;
  p2.Cf = out;
  p2.add0 = add0;
  p2.add1 = add1;
  return launch_gemm(ma, mb, p2, pair_tiles, stream);
}

bool build_tc_supported(int64_t V, int64_t D, int64_t Dr, const void* E, const void* W1, const void* W2,
                        const void* lut, const void* ws) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return false;
  if (D % 64 != 0 || Dr % 64 != 0 || V < 1 || V > (1LL << 31) - 1) return false;
  return aligned16(E) && aligned16(W1) && aligned16(W2) && aligned16(lut) && aligned16(ws) && encode_fn();
}

mole_status build_tc(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N, int64_t Dr,
                     int act, void* lut, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return build_tc_any(E, W1, W2, V, D, N, Dr, act, lut, nullptr, nullptr, ws, ws_bytes, stream);
}

// Training forward of the routed experts on the rows of Eu [M, D]: for every
// expert e, pre[e] = Eu . W1[e] (fp32), H[e] = act(pre[e]) (bf16), and
// Y[:, e, :] = H[e] . W2[e] (bf16, rows of N * D).  H and pre are [N, ld_rows,
// Dr]: expert e's matrix starts ld_rows * Dr elements after expert e-1's.
mole_status train_experts_tc(const void* Eu, const void* W1, const void* W2, int64_t M, int64_t ld_rows, int64_t D,
                             int N, int64_t Dr, int act, uint16_t* H, float* pre, uint16_t* Y, cudaStream_t stream) {
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const bool pair_tiles = M >= 2 * BM;
  const int mtile = pair_tiles ? 2 * BM : BM;
  CUtensorMap ma, mb;
  if (!make_map(&ma, Eu, D, M, 1, D * 2, M * D * 2, BM)) return MOLE_ERR_CUDA;
  if (!make_map(&mb, W1, Dr, D, N, Dr * 2, D * Dr * 2, BK)) return MOLE_ERR_CUDA;
  Params p1{};
  p1.M = (int)M;
  p1.N = (int)Dr;
  p1.K = (int)D;
  p1.a_e2 = 0;
  p1.b_e2 = 1;
  p1.act = act;
  p1.C = H;
  p1.ldc = Dr;
  p1.c_estride = ld_rows * Dr;
  p1.pre = pre;
  p1.pre_estride = ld_rows * Dr;
  p1.m_blocks = (int)((M + mtile - 1) / mtile);
  p1.n_blocks = (int)((Dr + BN - 1) / BN);
  p1.tiles = (int64_t)N * p1.m_blocks * p1.n_blocks;
  p1.err = err;
  mole_status st = launch_gemm(ma, mb, p1, pair_tiles, stream);
  if (st != MOLE_OK) return st;
  if (!make_map(&ma, H, Dr, M, N, Dr * 2, ld_rows * Dr * 2, BM)) return MOLE_ERR_CUDA;
  if (!make_map(&mb, W2, D, Dr, N, D * 2, Dr * D * 2, BK)) return MOLE_ERR_CUDA;
  Params p2{};
  p2.M = (int)M;
  p2.N = (int)D;
  p2.K = (int)Dr;
  p2.a_e2 = 1;
  p2.b_e2 = 1;
  p2.act = MOLE_ACT_IDENTITY;
  p2.C = Y;
  p2.ldc = (int64_t)N * D;
  p2.c_estride = D;
  p2.m_blocks = (int)((M + mtile - 1) / mtile);
  p2.n_blocks = (int)((D + BN - 1) / BN);
  p2.tiles = (int64_t)N * p2.m_blocks * p2.n_blocks;
  p2.err = err;
  return launch_gemm(ma, mb, p2, pair_tiles, stream);
}

namespace {

// dE[rowmap[u], :] += sum over the groups s, in order, of part[s][u, :]
// (each distinct id once).
__global__ void scatter_parts_kernel(const float* __restrict__ part, int64_t U, int64_t cap, int D, int S,
                                     const int* __restrict__ rowmap, float* dE) {
  const int64_t n = U * D;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t u = i / D, d = i - u * D;
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part[(int64_t)s * cap * D + i];
    dE[(int64_t)rowmap[u] * D + d] += acc;
  }
}

// Groups of experts for the dE contraction (a sum over all N experts' K):
// S groups (S divides N) of N / S experts each, one output tile set per
// group.  Fewer groups mean fewer partial sums to reduce but fewer tiles;
// pick the S with the least modelled time: waves of tiles over the CTA
// pairs, each wave as long as its tiles' K, plus a small cost per group.
int choose_groups(int N, int64_t tiles_per_group, int64_t units) {
  int best = 1;
  double best_cost = 1e300;
  for (int S = 1; S <= N; ++S) {
    if (N % S != 0) continue;
    const double waves = (double)((S * tiles_per_group + units - 1) / units);
    const double cost = waves * (double)(N / S) + 0.1 * S;
    if (cost < best_cost) {
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

}  // namespace

mole_status train_backward_tc(const uint16_t* dY, const uint16_t* H, const float* pre, const uint16_t* Eu,
                              const void* W1, const void* W2, int64_t U, int64_t cap, int64_t D, int N, int64_t Dr,
                              int act, uint16_t* dP, float* part, const int* rowmap, float* dW2, float* dW1,
                              float* dE, cudaStream_t stream) {
  if (U <= 0) return MOLE_OK;
  if (U > (1LL << 31) - 1 || D % 64 != 0 || Dr % 64 != 0) return MOLE_ERR_UNSUPPORTED;
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  const int64_t ND = (int64_t)N * D;
  CUtensorMap ma, mb;
  mole_status st;
  auto base = [&](Params& q, int64_t M, int64_t Nc, int64_t K, int n_out) {
    q.M = (int)M;
    q.N = (int)Nc;
    q.K = (int)K;
    const int mtile = M >= 2 * BM ? 2 * BM : BM;
    q.m_blocks = (int)((M + mtile - 1) / mtile);
    q.n_blocks = (int)((Nc + BN - 1) / BN);
    q.tiles = (int64_t)n_out * q.m_blocks * q.n_blocks;
    q.err = err;
    return M >= 2 * BM;  // CTA pairs once there are two 128-row blocks
  };
  if (dP != nullptr) {
    // dP[e] = bf16((dY_e . W2[e]^T) * act'(pre[e])): A = dY_e K-major (the
    // expert's block of each row), B = W2[e]^T K-major (W2[e] rows are k)
    if (!make_map(&ma, dY, ND, U, 1, ND * 2, U * ND * 2, BM) ||
        !make_map(&mb, W2, D, Dr, N, D * 2, Dr * D * 2, 128))
      return MOLE_ERR_CUDA;
    Params q{};
    const bool pr = base(q, U, Dr, D, N);
    q.a_e0 = (int)D;
    q.b_e2 = 1;
    q.act = act;
    q.C = dP;
    q.ldc = Dr;
    q.c_estride = cap * Dr;
    q.grad_pre = pre;
    q.pre_estride = cap * Dr;
    if ((st = launch_gemm<false, true>(ma, mb, q, pr, stream)) != MOLE_OK) return st;
  }
  if (dW2 != nullptr) {
    // dW2[e] += H[e]^T . dY_e: A = H[e]^T MN-major (H[e] rows are k of the
    // contraction), B = dY_e N-major
    if (!make_map(&ma, H, Dr, U, N, Dr * 2, cap * Dr * 2, BK) || !make_map(&mb, dY, ND, U, 1, ND * 2, U * ND * 2, BK))
      return MOLE_ERR_CUDA;
    Params q{};
    const bool pr = base(q, Dr, D, U, N);
    q.a_e2 = 1;
    q.b_e0 = (int)D;
    q.Cf = dW2;
    q.add0 = dW2;
    q.ldc = D;
    q.cf_estride = Dr * D;
    if ((st = launch_gemm<true, false>(ma, mb, q, pr, stream)) != MOLE_OK) return st;
  }
  if (dW1 != nullptr) {
    // dW1[e] += Eu^T . dP[e]: A = Eu^T MN-major, B = dP[e] N-major
    if (!make_map(&ma, Eu, D, U, 1, D * 2, U * D * 2, BK) || !make_map(&mb, dP, Dr, U, N, Dr * 2, cap * Dr * 2, BK))
      return MOLE_ERR_CUDA;
    Params q{};
    const bool pr = base(q, D, Dr, U, N);
    q.b_e2 = 1;
    q.Cf = dW1;
    q.add0 = dW1;
    q.ldc = Dr;
    q.cf_estride = D * Dr;
    if ((st = launch_gemm<true, false>(ma, mb, q, pr, stream)) != MOLE_OK) return st;
  }
  if (dE != nullptr) {
    // sum_e dP[e] . W1[e]^T: A = dP[e] K-major, B = W1[e]^T K-major (W1[e]
    // rows are d), the contraction over a group of experts' K ranges
    if (!make_map(&ma, dP, Dr, U, N, Dr * 2, cap * Dr * 2, BM) ||
        !make_map(&mb, W1, Dr, D, N, Dr * 2, D * Dr * 2, 128))
      return MOLE_ERR_CUDA;
    Params q{};
    const bool pr = base(q, U, D, Dr, 1);
    const int S = choose_groups(N, q.tiles, pr ? n_sm / 2 : n_sm);
    q.tiles *= S;
    q.a_e2 = 1;
    q.b_e2 = 1;
    q.k_experts = N / S;
    q.ldc = D;
    if (S == 1) {  // one group: straight into dE's rows
      q.Cf = dE;
      q.add0 = dE;
      q.c_rowmap = rowmap;
    } else {
      q.Cf = part;
      q.cf_estride = cap * D;
    }
    if ((st = launch_gemm<false, true>(ma, mb, q, pr, stream)) != MOLE_OK) return st;
    if (S > 1) {
      const int64_t n = U * D;
      const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)n_sm * 16));
      scatter_parts_kernel<<<grid, 256, 0, stream>>>(part, U, cap, (int)D, S, rowmap, dE);
      if (cudaGetLastError() != cudaSuccess) return MOLE_ERR_CUDA;
    }
  }
  return MOLE_OK;
}

mole_status build_tc_nf3(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N, int64_t Dr,
                         int act, uint8_t* codes, uint16_t* scales, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return build_tc_any(E, W1, W2, V, D, N, Dr, act, nullptr, codes, scales, ws, ws_bytes, stream);
}

// The build's two GEMMs per group of experts; the second writes either the
// bf16 table (lut) or, quantising in its epilogue, the NF3 codes and scales.
mole_status build_tc_any(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N, int64_t Dr,
                         int act, void* lut, uint8_t* codes, uint16_t* scales, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  const size_t per_expert = (size_t)V * Dr * 2;
  const int group = (int)std::min<size_t>((size_t)N, ws_bytes / per_expert);
  if (group < 1) return MOLE_ERR_WORKSPACE;
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const uint16_t* e16 = static_cast<const uint16_t*>(E);
  const uint16_t* w1 = static_cast<const uint16_t*>(W1);
  const uint16_t* w2 = static_cast<const uint16_t*>(W2);
  uint16_t* H = static_cast<uint16_t*>(ws);
  uint16_t* L = static_cast<uint16_t*>(lut);
  // CTA pairs (256-row tiles) once there are at least two 128-row blocks
  const bool pair_tiles = V >= 2 * BM;
  const int mtile = pair_tiles ? 2 * BM : BM;
  for (int e0 = 0; e0 < N; e0 += group) {
    const int g = std::min(group, N - e0);
    // GEMM1: H[e] = act(E . W1[e0 + e])
    CUtensorMap ma, mb;
    if (!make_map(&ma, e16, D, V, 1, D * 2, V * D * 2, BM)) return MOLE_ERR_CUDA;
    if (!make_map(&mb, w1 + (int64_t)e0 * D * Dr, Dr, D, g, Dr * 2, D * Dr * 2, BK)) return MOLE_ERR_CUDA;
    Params p1{};
    p1.M = (int)V;
    p1.N = (int)Dr;
    p1.K = (int)D;
    p1.a_e2 = 0;
    p1.b_e2 = 1;
    p1.act = act;
    p1.C = H;
    p1.ldc = Dr;
    p1.c_estride = V * Dr;
    p1.m_blocks = (int)((V + mtile - 1) / mtile);
    p1.n_blocks = (int)((Dr + BN - 1) / BN);
    p1.tiles = (int64_t)g * p1.m_blocks * p1.n_blocks;
    p1.err = err;
    mole_status st = launch_gemm(ma, mb, p1, pair_tiles, stream);
    if (st != MOLE_OK) return st;
    // GEMM2: LUT[:, e0 + e, :] = H[e] . W2[e0 + e]
    if (!make_map(&ma, H, Dr, V, g, Dr * 2, V * Dr * 2, BM)) return MOLE_ERR_CUDA;
    if (!make_map(&mb, w2 + (int64_t)e0 * Dr * D, D, Dr, g, D * 2, Dr * D * 2, BK)) return MOLE_ERR_CUDA;
    Params p2{};
    p2.M = (int)V;
    p2.N = (int)D;
    p2.K = (int)Dr;
    p2.a_e2 = 1;
    p2.b_e2 = 1;
    p2.act = MOLE_ACT_IDENTITY;
    if (codes != nullptr) {
      const int64_t nb = D / 64;  // NF3 blocks per row
      p2.codes = codes + (int64_t)e0 * nb * 24;
      p2.scales = scales + (int64_t)e0 * nb;
      p2.q_row = (int64_t)N * nb;
      p2.q_e = nb;
    } else {
      p2.C = L + (int64_t)e0 * D;
      p2.ldc = (int64_t)N * D;
      p2.c_estride = D;
    }
    p2.m_blocks = (int)((V + mtile - 1) / mtile);
    p2.n_blocks = (int)((D + BN - 1) / BN);
    p2.tiles = (int64_t)g * p2.m_blocks * p2.n_blocks;
    p2.err = err;
    st = launch_gemm(ma, mb, p2, pair_tiles, stream);
    if (st != MOLE_OK) return st;
  }
  return MOLE_OK;
}

}  // namespace mole
