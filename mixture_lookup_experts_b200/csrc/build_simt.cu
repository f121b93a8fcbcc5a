// build_simt.cu -- table build on CUDA cores (fp32 tables, and bf16 shapes the
// tensor-core path does not take).  MoLE page, 推理阶段: the embedding matrix is
// fed to every routed expert, LUT[v, j, :] = act(E[v] . W1[j]) . W2[j].
//
// Two batched tiled GEMMs per group of experts:
//   H[e] = act(E . W1[e])        (H rounded to bf16 for bf16 tables)
//   LUT[:, e, :] = H[e] . W2[e]  (row stride N * D)
// 64x64 output tiles, 16-deep k-slices in shared memory, 4x4 outputs per
// thread, fp32 accumulation.
#include "common.cuh"

namespace mole {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const TA* __restrict__ A, int64_t a_es, int64_t lda,
                                                        const TB* __restrict__ B, int64_t b_es, int64_t ldb,
                                                        TC* __restrict__ C, int64_t c_es, int64_t ldc, int M,
                                                        int Nn, int K, int act) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int e = blockIdx.z;
  A += e * a_es;
  B += e * b_es;
  C += e * c_es;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int mm = i / BK, kk = i % BK;
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? to_f32(A[(int64_t)gm * lda + gk]) : 0.f;
    }
    for (int i = threadIdx.x; i < BK * BN; i += 256) {
      const int kk = i / BN, nn = i % BN;
      const int gk = k0 + kk, gn = n0 + nn;
      Bs[kk][nn] = (gk < K && gn < Nn) ? to_f32(B[(int64_t)gk * ldb + gn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = Bs[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], b[jj], acc[i][jj]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int gn = n0 + tx * 4 + jj;
      if (gn >= Nn) continue;
      const float v = apply_act(act, acc[i][jj]);
      if constexpr (sizeof(TC) == 2)
        C[(int64_t)gm * ldc + gn] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
      else
        C[(int64_t)gm * ldc + gn] = v;
    }
  }
}

template <typename T>
mole_status run(const T* E, const T* W1, const T* W2, int64_t V, int64_t D, int N, int64_t Dr, int act,
                T* lut, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const size_t per_expert = (size_t)V * Dr * sizeof(T);
  const int group = (int)std::min<size_t>((size_t)N, ws_bytes / per_expert);
  if (group < 1) return MOLE_ERR_WORKSPACE;
  T* H = static_cast<T*>(ws);
  for (int e0 = 0; e0 < N; e0 += group) {
    const int g = std::min(group, N - e0);
    dim3 g1((unsigned)((Dr + BN - 1) / BN), (unsigned)((V + BM - 1) / BM), (unsigned)g);
    simt_gemm_kernel<T, T, T><<<g1, 256, 0, stream>>>(E, 0, D, W1 + (int64_t)e0 * D * Dr, D * Dr, Dr, H,
                                                      V * Dr, Dr, (int)V, (int)Dr, (int)D, act);
    dim3 g2((unsigned)((D + BN - 1) / BN), (unsigned)((V + BM - 1) / BM), (unsigned)g);
    simt_gemm_kernel<T, T, T><<<g2, 256, 0, stream>>>(H, V * Dr, Dr, W2 + (int64_t)e0 * Dr * D, Dr * D, D,
                                                      lut + (int64_t)e0 * D, D, (int64_t)N * D, (int)V,
                                                      (int)D, (int)Dr, MOLE_ACT_IDENTITY);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return MOLE_ERR_CUDA;
  }
  return MOLE_OK;
}

}  // namespace

mole_status build_simt(const void* E, const void* W1, const void* W2, int64_t V, int64_t D, int N,
                       int64_t Dr, int act, bool bf16, void* lut, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  if (V > 65535LL * BM) return MOLE_ERR_UNSUPPORTED;
  if (bf16)
    return run<uint16_t>(static_cast<const uint16_t*>(E), static_cast<const uint16_t*>(W1),
                         static_cast<const uint16_t*>(W2), V, D, N, Dr, act, static_cast<uint16_t*>(lut), ws,
                         ws_bytes, stream);
  return run<float>(static_cast<const float*>(E), static_cast<const float*>(W1), static_cast<const float*>(W2),
                    V, D, N, Dr, act, static_cast<float*>(lut), ws, ws_bytes, stream);
}

}  // namespace mole
