// plan.cu -- gather plan of a batch: the distinct token ids (ascending) and
// each token's slot among them, i.e. the set of table rows the batch has to
// fetch (MoLE page, 复杂度分析: per token only the expert-output vectors move).
//
// One CTA of 1024 threads keeps the id set as a bitmap in shared memory:
//   mark ids -> exclusive scan of per-word popcounts -> emit ids in order ->
//   slot[t] = prefix[word] + popcount(lower bits of that word).
// The result is deterministic and equals a sort + unique of the ids.
#include "common.cuh"

namespace mole {
namespace {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads) gather_plan_kernel(const int32_t* __restrict__ ids,
                                                                  int64_t T, int64_t V,
                                                                  int32_t* __restrict__ uniq,
                                                                  int32_t* __restrict__ n_uniq,
                                                                  int32_t* __restrict__ slot,
                                                                  unsigned* err) {
  extern __shared__ uint32_t sm[];
  const int nw = (int)((V + 31) >> 5);
  uint32_t* bits = sm;        // [nw]
  uint32_t* prefix = sm + nw; // [nw]
  __shared__ uint32_t warp_sums[kPlanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int w = tid; w < nw; w += kPlanThreads) bits[w] = 0u;
  __syncthreads();
  bool bad = false;
  for (int64_t t = tid; t < T; t += kPlanThreads) {
    const int32_t id = ids[t];
    if (id < 0 || (int64_t)id >= V) {
      bad = true;
      continue;
    }
    atomicOr(&bits[id >> 5], 1u << (id & 31));
  }
  if (bad) atomicOr(err, kErrIndex);
  __syncthreads();

  // exclusive scan of popcounts: each thread owns a contiguous chunk of words
  const int per = (nw + kPlanThreads - 1) / kPlanThreads;
  const int w0 = tid * per, w1 = min(nw, w0 + per);
  uint32_t local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(bits[w]);
  uint32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  uint32_t run = (warp > 0 ? warp_sums[warp - 1] : 0u) + incl - local;
  for (int w = w0; w < w1; ++w) {
    prefix[w] = run;
    run += __popc(bits[w]);
  }
  if (tid == 0) *n_uniq = (int32_t)warp_sums[kPlanThreads / 32 - 1];
  __syncthreads();

  for (int w = tid; w < nw; w += kPlanThreads) {
    uint32_t b = bits[w];
    uint32_t pos = prefix[w];
    while (b) {
      const int k = __ffs(b) - 1;
      uniq[pos++] = (w << 5) + k;
      b &= b - 1;
    }
  }
  for (int64_t t = tid; t < T; t += kPlanThreads) {
    const int32_t id = ids[t];
    if (id < 0 || (int64_t)id >= V) {
      slot[t] = -1;
      continue;
    }
    const int w = id >> 5;
    slot[t] = (int32_t)(prefix[w] + __popc(bits[w] & ((1u << (id & 31)) - 1u)));
  }
}

}  // namespace

constexpr int64_t kPlanMaxV = 524288;

mole_status gather_plan_launch(const int32_t* ids, int64_t T, int64_t V, int32_t* uniq,
                               int32_t* n_uniq, int32_t* slot, cudaStream_t stream) {
  if (V > kPlanMaxV) return MOLE_ERR_UNSUPPORTED;
  unsigned* err = error_word();
  if (!err) return MOLE_ERR_CUDA;
  const size_t smem = (size_t)2 * ((V + 31) >> 5) * sizeof(uint32_t);
  if (cudaFuncSetAttribute(gather_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOLE_ERR_CUDA;
  gather_plan_kernel<<<1, kPlanThreads, smem, stream>>>(ids, T, V, uniq, n_uniq, slot, err);
  return cuda_status(cudaGetLastError());
}

}  // namespace mole
