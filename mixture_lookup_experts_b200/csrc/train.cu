// train.cu -- one MoLE layer in training, forward and backward.  MoLE page,
// 训练阶段: during training the routed experts take the token's embedding row
// as input (not the previous layer's output), all N routed experts are
// active, and the router on the previous layer's output mixes them; the loss
// is the language-model loss alone.  Because a routed expert's input depends
// only on the token id, a batch needs the experts evaluated only on its
// distinct ids (a reading that follows from the page's setup; the page does
// not state it): the forward is the table build restricted to the batch's
// distinct embedding rows, then the inference combine over those rows.
//
// Forward (cache = what the backward needs; U = the batch's distinct ids):
//   Eu = E[distinct ids]                                  (row gather)
//   pre_j = Eu . W1_j, H_j = act(pre_j) (bf16), Y[:, j] = H_j . W2_j
//                                                         (the build's tcgen05 GEMMs)
//   out[t] = sum_j g_j(h[t]) Y[u(t), j]                   (the combine kernels)
// Backward of L with dL/dout = dout (all gradients accumulated, fp32):
//   g, dg_j = <dout[t], Y[u(t), j]>, dz = g (dg - <g, dg>)
//   dh[t] += dz[t] . Wr^T,  dWr += h^T dz                 (gate_grad_kernel; dwr_kernel per
//                                                          block of tokens, then dwr_reduce_kernel)
//   dY[u, j] = sum_{t: u(t) = u} g_j[t] dout[t]           (dy_kernel, one CTA per distinct id)
//   dpre_j = (dY_j . W2_j^T) * act'(pre_j)                (tcgen05 GEMM, derivative in its epilogue)
//   dW2_j += H_j^T dY_j,  dW1_j += Eu^T dpre_j             (tcgen05 GEMMs batched over the experts,
//                                                          fp32 gradients added in the epilogue)
//   dE[ids] += sum_j dpre_j . W1_j^T                      (tcgen05 GEMM whose contraction runs over
//                                                          the experts, rows scattered by id)
// The backward GEMMs are the table build's kernels with transposed operand
// forms (build_tc.cu); their bf16 operands dY and dpre are rounded from fp32.
#include "groups.cuh"

namespace mole {
namespace {

constexpr int kGradThreads = 256;
constexpr int kDwrTokens = 256;  // tokens per block of dwr_kernel

// The caller's cache buffer (cap = min(T, V) row capacity).
struct TrainCache {
  uint16_t* Eu;   // [cap, D] bf16
  uint16_t* Y;    // [cap, N, D] bf16
  uint16_t* H;    // [N, cap, Dr] bf16
  float* pre;     // [N, cap, Dr] fp32
  float* g;       // [T, N] gates
  float* dz;      // [T, N] logit gradients
  uint16_t* dYb;  // [cap, N, D] bf16: dL/dY by distinct id
  uint16_t* dP;   // [N, cap, Dr] bf16: dL/dpre
  float* dEu;     // [N, cap, D] fp32: partial sums of dL/dEu over groups of experts
  float* dWrp;    // [ceil(T / kDwrTokens), D, N] fp32: dWr per block of tokens
  int* U;         // one device int
  size_t total;
};

size_t carve_cache(void* base, int64_t T, int64_t V, int N, int64_t D, int64_t Dr, TrainCache* c) {
  const int64_t cap = std::min(T, V);
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  const size_t o_eu = take(2 * (size_t)cap * D);
  const size_t o_y = take(2 * (size_t)cap * N * D);
  const size_t o_h = take(2 * (size_t)N * cap * Dr);
  const size_t o_pre = take(4 * (size_t)N * cap * Dr);
  const size_t o_g = take(4 * (size_t)T * N);
  const size_t o_dz = take(4 * (size_t)T * N);
  const size_t o_dyb = take(2 * (size_t)cap * N * D);
  const size_t o_dp = take(2 * (size_t)N * cap * Dr);
  const size_t o_deu = take(4 * (size_t)N * cap * D);
  const size_t o_dwr = take(4 * (size_t)((T + kDwrTokens - 1) / kDwrTokens) * D * N);
  const size_t o_u = take(16);
  if (c != nullptr && base != nullptr) {
    uint8_t* b = static_cast<uint8_t*>(base);
    c->Eu = reinterpret_cast<uint16_t*>(b + o_eu);
    c->Y = reinterpret_cast<uint16_t*>(b + o_y);
    c->H = reinterpret_cast<uint16_t*>(b + o_h);
    c->pre = reinterpret_cast<float*>(b + o_pre);
    c->g = reinterpret_cast<float*>(b + o_g);
    c->dz = reinterpret_cast<float*>(b + o_dz);
    c->dYb = reinterpret_cast<uint16_t*>(b + o_dyb);
    c->dP = reinterpret_cast<uint16_t*>(b + o_dp);
    c->dEu = reinterpret_cast<float*>(b + o_deu);
    c->dWrp = reinterpret_cast<float*>(b + o_dwr);
    c->U = reinterpret_cast<int*>(b + o_u);
    c->total = off;
  }
  return off;
}

__device__ __forceinline__ float ld_bf16(const uint16_t* p) { return __uint_as_float((uint32_t)*p << 16); }

// Wr staged in shared memory as [D][NP] bf16 (experts past N zero), with 16
// bytes of padding after every 8 rows: a lane reads the 8 rows of its 8
// consecutive d, lanes 8 rows apart, so the padding spreads them over the banks.
__host__ __device__ __forceinline__ int wr_row(int d, int NP) { return d * NP + (d >> 3) * 8; }
__host__ __device__ __forceinline__ size_t wr_stage_bytes(int D, int NP) { return (size_t)(D * NP + (D >> 3) * 8) * 2; }

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// One warp per token: the gates (router logits h[t] . Wr in fp32, softmax),
// dg_j = <dout[t], Y[u(t), j]>, dz = g (dg - <g, dg>), and dh[t] += dz . Wr^T.
// Lane l takes d = 8l + 256i (16-byte loads of h, dout and the expert rows;
// Wr from the CTA's staged copy), then the partial sums are reduced across
// the warp.  Tokens with a bad id (dense index -1) get no gradient.
template <int NP>
__global__ void __launch_bounds__(kGradThreads) gate_grad_kernel(const GroupWs w, const uint16_t* __restrict__ h,
                                                                 const uint16_t* __restrict__ Wr,
                                                                 const uint16_t* __restrict__ Y,
                                                                 const float* __restrict__ dout, int64_t T, int N,
                                                                 int D, float* g_out, float* dz_out, float* dh) {
  extern __shared__ __align__(16) uint16_t wr_s[];
  for (int i = threadIdx.x; i < D * NP; i += kGradThreads) {
    const int d = i / NP, j = i - d * NP;
    wr_s[wr_row(d, NP) + j] = j < N ? Wr[(int64_t)d * N + j] : (uint16_t)0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kGradThreads / 32);
  for (int64_t t = (int64_t)blockIdx.x * (kGradThreads / 32) + (threadIdx.x >> 5); t < T; t += warps) {
    const int u = w.tok_uid[t];
    if (u < 0) continue;
    float z[NP], dg[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) z[j] = dg[j] = 0.f;
    const uint16_t* hr = h + t * D;
    const float* dr = dout + t * D;
    const uint16_t* yr = Y + (int64_t)u * N * D;
    for (int d0 = 8 * lane; d0 < D; d0 += 256) {
      float hf[8], of[8];
      unpack8(*reinterpret_cast<const uint4*>(hr + d0), hf);
      const float4 o0 = *reinterpret_cast<const float4*>(dr + d0);
      const float4 o1 = *reinterpret_cast<const float4*>(dr + d0 + 4);
      of[0] = o0.x; of[1] = o0.y; of[2] = o0.z; of[3] = o0.w;
      of[4] = o1.x; of[5] = o1.y; of[6] = o1.z; of[7] = o1.w;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint4* wr = reinterpret_cast<const uint4*>(wr_s + wr_row(d0 + e, NP));
#pragma unroll
        for (int q = 0; q < NP / 8; ++q) {
          float wf[8];
          unpack8(wr[q], wf);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) z[8 * q + jj] = fmaf(hf[e], wf[jj], z[8 * q + jj]);
        }
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        if (j < N) {
          float yf[8];
          unpack8(*reinterpret_cast<const uint4*>(yr + (int64_t)j * D + d0), yf);
#pragma unroll
          for (int e = 0; e < 8; ++e) dg[j] = fmaf(of[e], yf[e], dg[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NP; ++j)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        z[j] += __shfl_xor_sync(0xffffffffu, z[j], o);
        dg[j] += __shfl_xor_sync(0xffffffffu, dg[j], o);
      }
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < NP; ++j)
      if (j < N) m = fmaxf(m, z[j]);
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      z[j] = j < N ? expf(z[j] - m) : 0.f;
      sum += z[j];
    }
    float gdg = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      z[j] /= sum;  // the gate
      gdg = fmaf(z[j], dg[j], gdg);
    }
    float dz[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) dz[j] = z[j] * (dg[j] - gdg);
    if (lane < N) {
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j == lane) {
          g_out[t * N + j] = z[j];
          dz_out[t * N + j] = dz[j];
        }
    }
    if (dh != nullptr) {
      float* o = dh + t * D;
      for (int d0 = 8 * lane; d0 < D; d0 += 256) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4* wr = reinterpret_cast<const uint4*>(wr_s + wr_row(d0 + e, NP));
          acc[e] = 0.f;
#pragma unroll
          for (int q = 0; q < NP / 8; ++q) {
            float wf[8];
            unpack8(wr[q], wf);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) acc[e] = fmaf(dz[8 * q + jj], wf[jj], acc[e]);
          }
        }
        float4* o4 = reinterpret_cast<float4*>(o + d0);
        float4 a = o4[0], c = o4[1];
        a.x += acc[0]; a.y += acc[1]; a.z += acc[2]; a.w += acc[3];
        c.x += acc[4]; c.y += acc[5]; c.z += acc[6]; c.w += acc[7];
        o4[0] = a;
        o4[1] = c;
      }
    }
  }
}

// dWr over a block of kDwrTokens tokens: part[blockIdx.y][d][j] = sum over
// the block's tokens t (in order) of h[t, d] dz[t, j]; a thread per d.
template <int NP>
__global__ void __launch_bounds__(kGradThreads) dwr_kernel(const GroupWs w, const uint16_t* __restrict__ h,
                                                           const float* __restrict__ dz, int64_t T, int N, int D,
                                                           float* part) {
  __shared__ float dzs[kDwrTokens][NP];
  const int d = blockIdx.x * kGradThreads + threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.y * kDwrTokens;
  const int nt = (int)std::min<int64_t>(kDwrTokens, T - t0);
  for (int i = threadIdx.x; i < nt * NP; i += kGradThreads) {
    const int r = i / NP, j = i - r * NP;
    dzs[r][j] = (j < N && w.tok_uid[t0 + r] >= 0) ? dz[(t0 + r) * N + j] : 0.f;
  }
  __syncthreads();
  if (d >= D) return;
  float acc[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) acc[j] = 0.f;
  for (int r = 0; r < nt; ++r) {
    const float hv = ld_bf16(h + (t0 + r) * D + d);
#pragma unroll
    for (int j = 0; j < NP; ++j) acc[j] = fmaf(hv, dzs[r][j], acc[j]);
  }
  float* o = part + ((int64_t)blockIdx.y * D + d) * N;
#pragma unroll
  for (int j = 0; j < NP; ++j)
    if (j < N) o[j] = acc[j];
}

// dWr[i] += sum over the token blocks, in order, of part[b][i] (i = d N + j).
__global__ void dwr_reduce_kernel(const float* __restrict__ part, int n_blocks, int64_t n, float* dWr) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int b = 0; b < n_blocks; ++b) acc += part[(int64_t)b * n + i];
    dWr[i] += acc;
  }
}

// dY[u, j, d] = sum over the tokens t of id u, in list order, of
// g[t, j] dout[t, d], rounded to bf16 (the operand of the backward GEMMs).  Work unit = (work item, slice of kGradThreads
// consecutive d); only units of an id's first work item do work, over all of
// the id's tokens, so the sums do not depend on scheduling and a frequent id
// spreads over D / kGradThreads CTAs.  A thread holds the N sums of its d;
// tokens pass through shared memory kDyChunk at a time.  Every distinct id's
// rows are written (no clearing needed).
constexpr int kDyChunk = 64;

template <int NP>
__global__ void __launch_bounds__(kGradThreads) dy_kernel(const GroupWs w, const float* __restrict__ g,
                                                          const float* __restrict__ dout, int N, int D, uint16_t* dY) {
  __shared__ int toks[kDyChunk];
  __shared__ float gs[kDyChunk][NP];
  __shared__ int cnt_s;
  const int n_items = (int)ld_relaxed_u32(&w.ctl[kCtlItems]);
  const int n_slices = (D + kGradThreads - 1) / kGradThreads;
  const int64_t n_units = (int64_t)n_items * n_slices;
  for (int64_t unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
    const int it = (int)(unit / n_slices), sl = (int)(unit - (int64_t)it * n_slices);
    const int4 rec = w.items[it];  // {id, first list position, tokens, dense index}
    // the id's first item starts its range of the list (uniform over the CTA)
    if (rec.y > 0 && w.tok_uid[w.list[rec.y - 1]] == rec.w) continue;
    __syncthreads();  // the previous unit's readers of cnt_s, toks and gs are done
    if (threadIdx.x == 0) cnt_s = w.cnt[w.tok_slot[w.list[rec.y]]] + 1;
    __syncthreads();
    const int c = cnt_s;
    const int d = sl * kGradThreads + threadIdx.x;
    float acc[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) acc[j] = 0.f;
    for (int k0 = 0; k0 < c; k0 += kDyChunk) {
      const int n = c - k0 < kDyChunk ? c - k0 : kDyChunk;
      if (k0 > 0) __syncthreads();  // the previous chunk's readers are done
      if (threadIdx.x < n) toks[threadIdx.x] = w.list[rec.y + k0 + threadIdx.x];
      __syncthreads();
      for (int i = threadIdx.x; i < n * NP; i += kGradThreads) {
        const int k = i / NP, j = i - k * NP;
        gs[k][j] = j < N ? g[(int64_t)toks[k] * N + j] : 0.f;
      }
      __syncthreads();
      if (d < D) {
        int k = 0;
        for (; k + 4 <= n; k += 4) {  // four tokens' loads in flight
          float x[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) x[q] = dout[(int64_t)toks[k + q] * D + d];
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int j = 0; j < NP; ++j) acc[j] = fmaf(gs[k + q][j], x[q], acc[j]);
        }
        for (; k < n; ++k) {
          const float x = dout[(int64_t)toks[k] * D + d];
#pragma unroll
          for (int j = 0; j < NP; ++j) acc[j] = fmaf(gs[k][j], x, acc[j]);
        }
      }
    }
    if (d < D) {
      uint16_t* dst = dY + (int64_t)rec.w * N * D + d;
#pragma unroll
      for (int j = 0; j < NP; ++j)
        if (j < N) dst[(int64_t)j * D] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]));
    }
  }
}

unsigned grid_for(int64_t n, int per_block) {
  const int n_sm = num_sms();
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + per_block - 1) / per_block, (int64_t)n_sm * 16));
}

}  // namespace

size_t train_cache_bytes(int64_t T, int64_t V, int N, int64_t D, int64_t Dr) {
  return carve_cache(nullptr, T, V, N, D, Dr, nullptr);
}

mole_status train_forward(const void* groups, size_t gbytes, int64_t T, const void* h, const void* Wr, const void* E,
                          const void* W1, const void* W2, int64_t V, int N, int64_t D, int64_t Dr, int act,
                          float* out, void* cache, size_t cbytes, int32_t* n_distinct, cudaStream_t stream) {
  TrainCache c{};
  if (carve_cache(cache, T, V, N, D, Dr, &c) > cbytes) return MOLE_ERR_WORKSPACE;
  const int64_t cap = std::min(T, V);
  // the batch's distinct ids (one synchronisation: the GEMM sizes follow U)
  mole_status st = token_groups_count(groups, gbytes, T, N, c.U, stream);
  if (st != MOLE_OK) return st;
  int U = 0;
  if (cudaMemcpyAsync(&U, c.U, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return MOLE_ERR_CUDA;
  if (U < 0 || U > cap) return MOLE_ERR_CUDA;
  *n_distinct = U;
  if (U > 0) {
    st = gather_rows_by_uid(groups, gbytes, T, N, E, D * 2, V, c.Eu, cap, stream);
    if (st != MOLE_OK) return st;
    st = train_experts_tc(c.Eu, W1, W2, U, cap, D, N, Dr, act, c.H, c.pre, c.Y, stream);
    if (st != MOLE_OK) return st;
  }
  // the combine over the batch's expert rows, addressed by dense index
  return combine_offload(groups, gbytes, T, h, Wr, c.Y, (size_t)cap * N * D * 2, V, N, (int)D, true, false, out,
                         stream);
}

mole_status train_backward(const void* groups, size_t gbytes, int64_t T, const void* h, const void* Wr,
                           const void* W1, const void* W2, int64_t V, int N, int64_t D, int64_t Dr, int act,
                           const float* dout, void* cache, size_t cbytes, int32_t U, float* dh, float* dWr, float* dE,
                           float* dW1, float* dW2, cudaStream_t stream) {
  TrainCache c{};
  if (carve_cache(cache, T, V, N, D, Dr, &c) > cbytes) return MOLE_ERR_WORKSPACE;
  GroupWs w{};
  if (carve_ws(const_cast<void*>(groups), T, padded_experts(N), &w) > gbytes) return MOLE_ERR_WORKSPACE;
  const int64_t cap = std::min(T, V);
  if (U < 0 || U > cap) return MOLE_ERR_ARG;
  const uint16_t* h16 = static_cast<const uint16_t*>(h);
  const uint16_t* wr16 = static_cast<const uint16_t*>(Wr);
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  // gates, logit gradients, dh (Wr staged per CTA: a few CTAs per SM)
  {
    const int NP = N <= 8 ? 8 : N <= 16 ? 16 : 32;
    const size_t smem = wr_stage_bytes((int)D, NP);
    auto kern = N <= 8 ? gate_grad_kernel<8> : N <= 16 ? gate_grad_kernel<16> : gate_grad_kernel<32>;
    if (smem > 227 * 1024) return MOLE_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOLE_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGradThreads, smem) != cudaSuccess || occ < 1)
      return MOLE_ERR_UNSUPPORTED;
    const unsigned gg = (unsigned)std::min<int64_t>((T + 7) / 8, (int64_t)n_sm * occ);
    kern<<<gg, kGradThreads, smem, stream>>>(w, h16, wr16, c.Y, dout, T, N, (int)D, c.g, c.dz, dh);
    if (cudaGetLastError() != cudaSuccess) return MOLE_ERR_CUDA;
  }
  if (dWr != nullptr) {
    const dim3 gw((unsigned)((D + kGradThreads - 1) / kGradThreads), (unsigned)((T + kDwrTokens - 1) / kDwrTokens));
    if (N <= 8)
      dwr_kernel<8><<<gw, kGradThreads, 0, stream>>>(w, h16, c.dz, T, N, (int)D, c.dWrp);
    else if (N <= 16)
      dwr_kernel<16><<<gw, kGradThreads, 0, stream>>>(w, h16, c.dz, T, N, (int)D, c.dWrp);
    else
      dwr_kernel<32><<<gw, kGradThreads, 0, stream>>>(w, h16, c.dz, T, N, (int)D, c.dWrp);
    dwr_reduce_kernel<<<grid_for(D * N, 256), 256, 0, stream>>>(c.dWrp, (int)gw.y, D * N, dWr);
    if (cudaGetLastError() != cudaSuccess) return MOLE_ERR_CUDA;
  }
  if (U == 0 || (dE == nullptr && dW1 == nullptr && dW2 == nullptr)) return MOLE_OK;
  // dY by distinct id (bf16), then the expert GEMMs
  if (N <= 8)
    dy_kernel<8><<<(unsigned)n_sm * 4, kGradThreads, 0, stream>>>(w, c.g, dout, N, (int)D, c.dYb);
  else if (N <= 16)
    dy_kernel<16><<<(unsigned)n_sm * 4, kGradThreads, 0, stream>>>(w, c.g, dout, N, (int)D, c.dYb);
  else
    dy_kernel<32><<<(unsigned)n_sm * 4, kGradThreads, 0, stream>>>(w, c.g, dout, N, (int)D, c.dYb);
  if (cudaGetLastError() != cudaSuccess) return MOLE_ERR_CUDA;
  const bool need_dp = dW1 != nullptr || dE != nullptr;
  return train_backward_tc(c.dYb, c.H, c.pre, c.Eu, W1, W2, U, cap, D, N, Dr, act, need_dp ? c.dP : nullptr, c.dEu,
                           w.uid_id, dW2, dW1, dE, stream);
  return MOLE_OK;
}

}  // namespace mole
