// router_tc.cu -- the router of a prefill batch on the tcgen05 tensor cores
// (MoLE page, 训练阶段: the gates are a softmax over all routed experts of the
// hidden state times the router weight), taken by the NF3-table calls; the
// bf16-table calls route with the mma.sync router arithmetic throughout.
//
// z[T, 16] = h[T, D] . Wr[D, 16] is a skinny GEMM bound by reading h (2D bytes
// per token).  One CTA per SM, persistent over 128-token tiles:
//   warp 0     TMA producer (one lane): the h box 64(d) x rows(tokens) with
//              128-byte swizzle and the Wr box 16(j) x 64(d) with 32-byte
//              swizzle -- Wr is read in its own [D, N] layout as the N-major
//              B operand -- into an 8-stage ring of 18 KB;
//   warp 1     TMEM owner + MMA issuer (one lane): tcgen05.mma kind::f16,
//              M=128 N=16 K=16, fp32 accumulators double-buffered in 32 TMEM
//              columns;
//   warps 2-5  epilogue, one token per thread (its TMEM lane): 16 logits by
//              tcgen05.ld, max-subtracted softmax, and the 16 gates stored
//              either in the token's output row (where the gather kernel of
//              mole_lookup_combine picks them up) or at the token's list
//              position of a token grouping (mole_lookup_combine_groups).
// The h stream keeps up to 8 x 16 KB in flight per SM without tying up
// registers, so the router runs near the HBM rate.
//
// Every wait is bounded; a wait that runs out sets the device error word, the
// roles leave their loops, outstanding copies and MMAs are drained with
// bounded waits and TMEM is released before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace mole {
namespace {

constexpr int RM = 128, RK = 64, RN = 16, RSTAGES = 8, RBOX = 1;
constexpr int RKS = RK * RBOX;              // hidden dims per stage
constexpr int RA_BOX = RM * RK * 2;          // one 16 KB h box (64 dims x 128 tokens)
constexpr int RA_STAGE = RA_BOX * RBOX;
constexpr int RB_STAGE = RKS * RN * 2;       // Wr rows of the stage
constexpr int kRThreads = 6 * 32;
constexpr int kREpiWarps = 4;
constexpr int kRSmem = 1024 /*alignment slack*/ + RSTAGES * (RA_STAGE + RB_STAGE) + 256 /*barriers*/;
constexpr uint32_t kRTmemCols = 32;  // two 16-column accumulators
constexpr bool kRotateK = true;

// Instruction descriptor, kind::f16: D fp32 (bit 4), A bf16 (bits 7-9) K-major,
// B bf16 (bits 10-12) N-major (bit 16), N/8 at bits 17-22, M/16 at bits 24-28.
constexpr uint32_t kRIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(RN >> 3) << 17) |
                             ((uint32_t)(RM >> 4) << 24);

enum RouterSink { kSinkOutRows = 0, kSinkGrouped = 1 };

struct RtArgs {
  int64_t T;
  int D;
  int rows;  // tokens per tile (<= RM; the MMA still runs M = RM, extra lanes are dropped)
  int64_t tiles;
  float* out;           // [T, D]
  const int* tok_pos;   // grouped: list position of each token (-1: bad id)
  float* gates;         // grouped: [T][16] by list position
  unsigned* err;
};

__device__ __forceinline__ void rt_tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                               int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void rt_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void rt_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (sm_100 layout version 1); layout 2 =
// 128-byte swizzle, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t rt_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

__device__ __forceinline__ void rt_umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kRIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void rt_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void rt_tmem_ld16(uint32_t taddr, float (&z)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) z[i] = __uint_as_float(r[i]);
}

template <int kSink>
__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w,
                     const RtArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + RSTAGES * RA_STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + RSTAGES * RB_STAGE);
  uint64_t* empty = full + RSTAGES;
  uint64_t* tfull = empty + RSTAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kREpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kRTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  rt_fence_before();
  __syncthreads();
  rt_fence_after();
  // under a programmatic dependent launch: let the next kernel get scheduled,
  // then wait for the previous one (it may have produced h or Wr, or still
  // read what this kernel writes)
  pdl_trigger();
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;
  const int kblocks = (p.D + RKS - 1) / RKS;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t it = 0;
      bool ok = true;
      const uint32_t box_bytes = (uint32_t)p.rows * RK * 2;
      for (int64_t tile = blockIdx.x; ok && tile < p.tiles; tile += gridDim.x) {
        const int k0 = kRotateK ? (int)(tile % kblocks) : 0;
        for (int i = 0; i < kblocks; ++i, ++it) {
          const int kb = k0 + i < kblocks ? k0 + i : k0 + i - kblocks;
          const uint32_t s = it % RSTAGES, ph = (it / RSTAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort, p.err)) {
            ok = false;
            break;
          }
          const int nbox = min(RBOX, (p.D - kb * RKS + RK - 1) / RK);
          mbar_expect_tx(&full[s], (uint32_t)nbox * box_bytes + RB_STAGE);
          for (int b = 0; b < nbox; ++b)
            rt_tma_load_3d(sA + s * RA_STAGE + b * RA_BOX, &map_h, &full[s], kb * RKS + b * RK, (int)(tile * p.rows),
                           0);
          rt_tma_load_3d(sB + s * RB_STAGE, &map_w, &full[s], 0, kb * RKS, 0);
        }
      }
      const uint32_t first = it > (uint32_t)RSTAGES ? it - RSTAGES : 0u;
      for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % RSTAGES], (i / RSTAGES) & 1u);
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
        rt_fence_after();
        const uint32_t d_tmem = tmem_base + acc * RN;
        const int k0 = kRotateK ? (int)(tile % kblocks) : 0;
        for (int i = 0; i < kblocks; ++i, ++it) {
          const int kb = k0 + i < kblocks ? k0 + i : k0 + i - kblocks;
          const uint32_t s = it % RSTAGES, ph = (it / RSTAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort, p.err)) {
            ok = false;
            break;
          }
          rt_fence_after();
          const uint32_t a0 = smem_u32(sA + s * RA_STAGE), b0 = smem_u32(sB + s * RB_STAGE);
          const int nk = min(RKS, p.D - kb * RKS) / 16;
#pragma unroll
          for (int k = 0; k < RKS / 16; ++k) {
            if (k >= nk) break;
            // A (h): K-major, 128-byte rows; advance 16 elements (32 B) inside the swizzle atom,
            // and a whole 16 KB box every 64 elements.
            // B (Wr): N-major, 32-byte rows of 16 experts; 8-row atoms of 256 B; advance 16 rows (512 B).
            rt_umma(d_tmem, rt_desc(a0 + (k >> 2) * RA_BOX + 32 * (k & 3), 16, 1024, 2),
                    rt_desc(b0 + 512 * k, 0, 256, 6), (i | k) != 0);
          }
          issued = true;
          rt_commit(&empty[s]);
        }
        if (ok) rt_commit(&tfull[acc]);
      }
      if (!ok && issued) {
        rt_commit(drain);
        mbar_drain(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quad = warp & 3;  // the TMEM lanes this warp may access
    uint32_t tl = 0;
    for (int64_t tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++tl) {
      const uint32_t acc = tl & 1u, aph = (tl >> 1) & 1u;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&tfull[acc], aph, abort, p.err);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      rt_fence_after();
      float z[16];
      rt_tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + acc * RN, z);
      rt_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      const int r = quad * 32 + lane;
      const int64_t t = tile * p.rows + r;
      if (r >= p.rows || t >= p.T) continue;
      float m = z[0];
#pragma unroll
      for (int j = 1; j < 16; ++j) m = fmaxf(m, z[j]);
      float e[16], sum = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        e[j] = expf(z[j] - m);
        sum += e[j];
      }
      float4* dst;
      if (kSink == kSinkOutRows) {
        dst = reinterpret_cast<float4*>(p.out + t * p.D);
      } else {
        const int pos = p.tok_pos[t];
        if (pos < 0) {  // a bad id: NaN output row
          atomicOr(p.err, kErrIndex);
          float4* o = reinterpret_cast<float4*>(p.out + t * p.D);
          for (int d = 0; d < p.D / 4; ++d) __stcs(o + d, make_float4(NAN, NAN, NAN, NAN));
          continue;
        }
        dst = reinterpret_cast<float4*>(p.gates + (int64_t)pos * RN);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_float4(e[4 * q] / sum, e[4 * q + 1] / sum, e[4 * q + 2] / sum, e[4 * q + 3] / sum);
    }
  }

  __syncthreads();
  if (warp == 1) {
    rt_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kRTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 rt_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) == cudaSuccess &&
        res == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(q);
  }
  return fn;
}

// 3-D bf16 tensor map {d0 (contiguous), d1, 1}, box {box0, box1, 1}, zero fill
// out of bounds.
bool rt_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t s1_bytes, uint32_t box0,
            uint32_t box1, CUtensorMapSwizzle swz) {
  auto fn = rt_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, 1};
  cuuint64_t strides[2] = {s1_bytes, s1_bytes};  // the third dimension has extent 1
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tokens per tile: as many rounds of RM-token tiles as the batch needs over
// the SMs, then the rows evened out over them (a multiple of 16), so that the
// last round does not leave SMs idle -- 16384 tokens on 148 SMs take 147
// tiles of 112 rows rather than 128 tiles of 128.
int router_tile_rows(int64_t T, int n_sm) {
  const int64_t rounds = (T + (int64_t)n_sm * RM - 1) / ((int64_t)n_sm * RM);
  const int64_t per = (T + (int64_t)n_sm * rounds - 1) / ((int64_t)n_sm * rounds);
  return (int)std::min<int64_t>(RM, (per + 15) / 16 * 16);
}

}  // namespace

bool router_tc_supported(int64_t T, int N, int64_t D, const void* h, const void* Wr) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return false;
  // one CTA per 128-token tile: below about 3/4 of a tile per SM the
  // 16-token-tile router of combine_common.cuh spreads the batch wider
  const int n_sm = num_sms();
  if (n_sm <= 0 || (T + RM - 1) / RM < (int64_t)n_sm * 3 / 4) return false;
  return N == RN && T <= INT32_MAX && D >= 16 && D % 16 == 0 && aligned16(h) && aligned16(Wr) &&
         rt_encode_fn() != nullptr;
}

mole_status router_tc_launch(const void* h, const void* Wr, int64_t T, int64_t D, bool grouped, float* out,
                             const int* tok_pos, float* gates, cudaStream_t stream) {
  CUtensorMap mh, mw;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  const int rows = router_tile_rows(T, n_sm);
  if (!rt_map(&mh, h, (uint64_t)D, (uint64_t)T, (uint64_t)D * 2, RK, (uint32_t)rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !rt_map(&mw, Wr, RN, (uint64_t)D, RN * 2, RN, RKS, CU_TENSOR_MAP_SWIZZLE_32B))
    return MOLE_ERR_CUDA;
  static bool attr_set[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOLE_ERR_CUDA;
  auto kern = grouped ? router_tc_kernel<kSinkGrouped> : router_tc_kernel<kSinkOutRows>;
  if (!attr_set[dev][grouped]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem) != cudaSuccess)
      return MOLE_ERR_CUDA;
    attr_set[dev][grouped] = true;
  }
  RtArgs p{};
  p.T = T;
  p.D = (int)D;
  p.rows = rows;
  p.tiles = (T + rows - 1) / rows;
  p.out = out;
  p.tok_pos = tok_pos;
  p.gates = gates;
  p.err = error_word();
  if (!p.err) return MOLE_ERR_CUDA;
  const unsigned grid = (unsigned)std::min<int64_t>(p.tiles, n_sm);
  return cuda_status(launch_pdl(kern, grid, kRThreads, kRSmem, stream, mh, mw, p));
}

}  // namespace mole
