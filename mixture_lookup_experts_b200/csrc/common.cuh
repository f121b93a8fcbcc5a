// common.cuh -- internal helpers shared by the libmole translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <utility>
#include <stdint.h>

#include <algorithm>

#include "mole.h"

namespace mole {

// Bits of the per-device error word (set by kernels with atomicOr).
enum : unsigned {
  kErrIndex = 1u,    // a token id outside [0, V)
  kErrTimeout = 2u,  // a bounded device-side wait gave up
  kErrGrouping = 4u, // a grouping used on a device other than the one it was built for
};

// Device address of this device's error word (resolved once per device).
unsigned* error_word();

// Number of SMs of the current device (cached per device).
int num_sms();

// Turns a launch / runtime error into a status.
inline mole_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOLE_OK : MOLE_ERR_CUDA; }

// Launches `kernel` with programmatic stream serialization: it may begin
// while the previous kernel in the stream finishes (the kernel waits with
// griddepcontrol.wait before touching that kernel's results).
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// ---- device helpers -------------------------------------------------------

// bf16 pair packed in a 32-bit word -> the two fp32 values (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 16-byte read-only load that does not allocate in L1 (streamed table rows).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

// 16-byte store with an evict-first hint (outputs are written once).
__device__ __forceinline__ void stg_stream(void* p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}

}  // namespace mole

namespace mole {

// GELU(u) = u * Phi(u).  Phi through the complementary error function of
// x = |u|/sqrt(2), evaluated with Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26 (erfc(x) = t(a1 + t(a2 + ... + t a5)) exp(-x^2),
// t = 1/(1 + p x), absolute error <= 1.5e-7): Phi(u) = erfc(x)/2 for u < 0 and
// 1 - erfc(x)/2 for u >= 0, so neither side subtracts nearly equal numbers.
// About 15 instructions, two of them on the special-function unit.
__device__ __forceinline__ float gelu_as7126(float u) {
  const float x = fabsf(u) * 0.7071067811865476f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, x, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  const float half_erfc = 0.5f * (poly * t) * __expf(-x * x);
  return u * (u >= 0.f ? 1.0f - half_erfc : half_erfc);
}

// Expert FFN activation with the kind fixed at compile time (no branch in
// per-element loops).
template <int ACT>
__device__ __forceinline__ float act_t(float x) {
  if constexpr (ACT == MOLE_ACT_GELU_ERF) {
    return gelu_as7126(x);
  } else if constexpr (ACT == MOLE_ACT_GELU_TANH) {
    const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
    return 0.5f * x * (1.f + tanhf(u));
  } else if constexpr (ACT == MOLE_ACT_RELU) {
    return x > 0.f ? x : 0.f;
  } else if constexpr (ACT == MOLE_ACT_SILU) {
    return __fdividef(x, 1.f + __expf(-x));
  } else {
    return x;
  }
}

// Derivative of the expert activation at u, kind fixed at compile time (the
// training backward's dL/dpre = dL/dH * act'(pre)).  GELU: Phi(u) + u phi(u),
// Phi through the same Abramowitz & Stegun 7.1.26 erfc as the forward.
template <int ACT>
__device__ __forceinline__ float act_grad_t(float u) {
  if constexpr (ACT == MOLE_ACT_GELU_ERF) {
    const float x = fabsf(u) * 0.7071067811865476f;
    const float t = __fdividef(1.0f, fmaf(0.3275911f, x, 1.0f));
    float poly = fmaf(1.061405429f, t, -1.453152027f);
    poly = fmaf(poly, t, 1.421413741f);
    poly = fmaf(poly, t, -0.284496736f);
    poly = fmaf(poly, t, 0.254829592f);
    const float e = __expf(-x * x);                      // exp(-u^2 / 2)
    const float half_erfc = 0.5f * (poly * t) * e;
    const float Phi = u >= 0.f ? 1.0f - half_erfc : half_erfc;
    return fmaf(u * 0.3989422804014327f, e, Phi);       // + u phi(u), phi(u) = e / sqrt(2 pi)
  } else if constexpr (ACT == MOLE_ACT_GELU_TANH) {
    const float c = 0.7978845608028654f;
    const float th = tanhf(c * fmaf(0.044715f * u, u * u, u));
    return 0.5f * (1.f + th) + 0.5f * u * (1.f - th * th) * c * fmaf(3.f * 0.044715f, u * u, 1.f);
  } else if constexpr (ACT == MOLE_ACT_RELU) {
    return u > 0.f ? 1.f : 0.f;
  } else if constexpr (ACT == MOLE_ACT_SILU) {
    const float sg = __fdividef(1.f, 1.f + __expf(-u));
    return sg * fmaf(u, 1.f - sg, 1.f);
  } else {
    return 1.f;
  }
}

// Expert FFN activation (reading of the page's "GELU FFN": exact GELU x*Phi(x)).
__device__ __forceinline__ float apply_act(int act, float x) {
  switch (act) {
    case MOLE_ACT_GELU_ERF: return gelu_as7126(x);
    case MOLE_ACT_GELU_TANH: {
      const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);  // sqrt(2/pi) (x + 0.044715 x^3)
      return 0.5f * x * (1.f + tanhf(u));
    }
    case MOLE_ACT_RELU: return x > 0.f ? x : 0.f;
    case MOLE_ACT_SILU: return __fdividef(x, 1.f + __expf(-x));
    default: return x;
  }
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Build-path entry points (build_simt.cu / build_tc.cu).
mole_status build_simt(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N,
                       int64_t Dr, int act, bool bf16, void* lut, void* ws, size_t ws_bytes,
                       cudaStream_t stream);
bool build_tc_supported(int64_t V, int64_t D, int64_t Dr, const void* E, const void* W1,
                        const void* W2, const void* lut, const void* ws);
mole_status build_tc(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N,
                     int64_t Dr, int act, void* lut, void* ws, size_t ws_bytes, cudaStream_t stream);
// The routed experts of a training step on the rows of Eu (build_tc.cu).
mole_status train_experts_tc(const void* Eu, const void* W1, const void* W2, int64_t M, int64_t ld_rows, int64_t D,
                             int N, int64_t Dr, int act, uint16_t* H, float* pre, uint16_t* Y, cudaStream_t stream);
// The four expert GEMMs of a training step's backward (build_tc.cu), on the
// U distinct ids' rows (matrices of `cap` rows per expert, the first U used):
//   dP[e]  = bf16((dY[:, e, :] . W2[e]^T) * act'(pre[e]))       dY [cap, N, D] bf16
//   dW2[e] += H[e]^T . dY[:, e, :]                              H, pre, dP [N, cap, Dr]
//   dW1[e] += Eu^T . dP[e]                                      Eu [cap, D] bf16
//   dE[rowmap[u]] += sum_e dP[e][u] . W1[e]^T                   part [N, cap, D] fp32 scratch
// Each is one tcgen05 GEMM launch (the last plus a reduction over groups of
// experts when the sum is split); any of dW2, dW1, dE may be null.
mole_status train_backward_tc(const uint16_t* dY, const uint16_t* H, const float* pre, const uint16_t* Eu,
                              const void* W1, const void* W2, int64_t U, int64_t cap, int64_t D, int N, int64_t Dr,
                              int act, uint16_t* dP, float* part, const int* rowmap, float* dW2, float* dW1,
                              float* dE, cudaStream_t stream);
// The build with the NF3 quantiser in the second GEMM's epilogue (no bf16 table).
mole_status build_tc_nf3(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N, int64_t Dr,
                         int act, uint8_t* codes, uint16_t* scales, void* ws, size_t ws_bytes, cudaStream_t stream);

// Shared-expert FFN on the tensor cores (build_tc.cu): out = act(h . W1s) . W2s
// + add0 + add1 (fp32), the hidden activation rounded to bf16 in `ws`.
bool shared_ffn_tc_supported(int64_t T, int64_t D, int64_t Ds, const void* h, const void* W1s, const void* W2s,
                             const void* add0, const void* add1, const void* out, const void* ws);
mole_status shared_ffn_tc(const void* h, const void* W1s, const void* W2s, int64_t T, int64_t D, int64_t Ds, int act,
                          const float* add0, const float* add1, float* out, void* ws, size_t ws_bytes,
                          cudaStream_t stream);
// Combine / NF3 / plan entry points (combine.cu / plan.cu).
mole_status combine_dispatch(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                             const void* table, const uint16_t* scales, int64_t V, int N, int D,
                             bool bf16_inputs, int table_kind, float* out, cudaStream_t stream);
mole_status nf3_quantize_launch(const void* lut, int64_t V, int N, int64_t D, uint8_t* codes,
                                uint16_t* scales, cudaStream_t stream);
// Router of a prefill batch on the tensor cores (router_tc.cu; N == 16):
// gates into the tokens' output rows, or (grouped) at their list positions.
bool router_tc_supported(int64_t T, int N, int64_t D, const void* h, const void* Wr);
mole_status router_tc_launch(const void* h, const void* Wr, int64_t T, int64_t D, bool grouped, float* out,
                             const int* tok_pos, float* gates, cudaStream_t stream);
// Id-grouped combine (grouped.cu): the grouping of a batch's tokens by id
// (built once per batch), one layer's combine with it, and both in one call;
// the combines fall back to combine_dispatch where the grouped kernels do not
// apply.
size_t token_groups_bytes(int64_t T, int N);
mole_status token_groups_build(const int32_t* ids, int64_t T, int64_t V, int N, void* buf, size_t bytes,
                               cudaStream_t stream);
mole_status combine_groups(const void* buf, size_t bytes, int64_t T, const void* h, const void* Wr,
                           const void* table, const uint16_t* scales, bool nf3, int N, int D, float* out,
                           cudaStream_t stream);
mole_status combine_grouped_dispatch(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                     const void* table, const uint16_t* scales, int64_t V, int N, int D,
                                     bool bf16_inputs, int table_kind, float* out, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);
// Offloaded table (grouped.cu): the batch's distinct row blocks staged from a
// table the device reads in place (pinned host memory), and the combine that
// reads the staging buffer.
// Largest batch a token grouping (and so an offloaded-table call) takes.
constexpr int64_t kMaxOffloadT = int64_t(1) << 30;
size_t offload_staging_bytes(int64_t T, int64_t V, int N, int D, int elem_bytes, bool nf3);
mole_status offload_stage(const void* buf, size_t bytes, int64_t T, const void* table, const void* scales,
                          int64_t V, int N, int D, int elem_bytes, bool nf3, void* staging, size_t staging_bytes,
                          int* n_rows, cudaStream_t stream);
mole_status combine_offload(const void* buf, size_t bytes, int64_t T, const void* h, const void* Wr,
                            const void* staging, size_t staging_bytes, int64_t V, int N, int D, bool bf16_inputs,
                            bool nf3, float* out, cudaStream_t stream);
// The batch's distinct-id count (device int) and the rows of a table for its
// distinct ids by dense index (grouped.cu; training).
mole_status token_groups_count(const void* buf, size_t bytes, int64_t T, int N, int* dst, cudaStream_t stream);
mole_status gather_rows_by_uid(const void* buf, size_t bytes, int64_t T, int N, const void* table, int64_t row_bytes,
                               int64_t V, void* dst, int64_t cap, cudaStream_t stream);
// Training (train.cu): the cache size, the forward (experts on the batch's
// distinct ids, then the combine) and the backward.
size_t train_cache_bytes(int64_t T, int64_t V, int N, int64_t D, int64_t Dr);
mole_status train_forward(const void* groups, size_t gbytes, int64_t T, const void* h, const void* Wr, const void* E,
                          const void* W1, const void* W2, int64_t V, int N, int64_t D, int64_t Dr, int act,
                          float* out, void* cache, size_t cbytes, int32_t* n_distinct, cudaStream_t stream);
mole_status train_backward(const void* groups, size_t gbytes, int64_t T, const void* h, const void* Wr,
                           const void* W1, const void* W2, int64_t V, int N, int64_t D, int64_t Dr, int act,
                           const float* dout, void* cache, size_t cbytes, int32_t U, float* dh, float* dWr, float* dE,
                           float* dW1, float* dW2, cudaStream_t stream);
void nf3_tables(uint16_t levels[8], float mid[7]);
mole_status gather_plan_launch(const int32_t* ids, int64_t T, int64_t V, int32_t* uniq,
                               int32_t* n_uniq, int32_t* slot, cudaStream_t stream);

}  // namespace mole

namespace mole {

// ---- mbarrier helpers with bounded waits (shared by the TMA pipelines) ----
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // a wait gives up after 4 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Programmatic dependent launch (kernels launched with the programmatic
// stream serialization attribute may start while the previous kernel in the
// stream is still running): pdl_trigger lets the next kernel start early;
// pdl_wait blocks until the previous kernel has completed and its memory is
// visible.  Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps in the barrier unit (issuing nothing) until the phase completes or
// about hint_ns have passed, instead of spinning on the scheduler.
__device__ __forceinline__ bool mbar_test_sleep(uint64_t* b, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kSuspendHintNs = 20000;

// Waits for the phase with the given parity to complete.  Gives up (returns
// false) when *abort is set by another role or after kWaitLimitNs, in which
// case it sets *abort and the device error word.
static __device__ __noinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort, unsigned* err) {
  if (mbar_test(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_test(b, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
}

// Bounded wait used while draining after an abort (ignores the abort flag).
static __device__ __noinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_test(b, parity))
    if (globaltimer() - t0 > kWaitLimitNs) return;
}

}  // namespace mole
