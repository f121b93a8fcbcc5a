// api.cu -- extern "C" entry points of libmole (declared in include/mole.h).
// Validates arguments on the host, then enqueues the kernels on the caller's
// stream.  No entry point allocates device memory.
#include "common.cuh"

namespace {

bool valid_dtype(mole_dtype dt) { return dt == MOLE_F32 || dt == MOLE_BF16; }
bool valid_act(mole_act a) { return a >= MOLE_ACT_GELU_ERF && a <= MOLE_ACT_IDENTITY; }
size_t dtype_size(mole_dtype dt) { return dt == MOLE_BF16 ? 2 : 4; }

mole_status check_device() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOLE_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOLE_ERR_NO_DEVICE;
  return major == 10 ? MOLE_OK : MOLE_ERR_NO_DEVICE;
}

// Shared checks of the two combine entry points.
mole_status check_combine(const int32_t* ids, int64_t T, const void* h, const void* Wr, const void* table,
                          int64_t V, int32_t N, int64_t D, float* out) {
  if (T < 0 || V <= 0 || V > INT32_MAX || N <= 0 || D <= 0 || D > (1 << 20)) return MOLE_ERR_ARG;
  if (T > 0 && (!ids || !h || !Wr || !table || !out)) return MOLE_ERR_ARG;
  if (N > 32) return MOLE_ERR_UNSUPPORTED;
  if (T > ((int64_t)1 << 40)) return MOLE_ERR_UNSUPPORTED;
  if (!mole::aligned16(h) || !mole::aligned16(out)) return MOLE_ERR_ALIGN;
  return MOLE_OK;
}

}  // namespace

extern "C" size_t mole_build_lut_workspace(int64_t V, int64_t D, int32_t N, int64_t Dr, mole_dtype dt,
                                           int32_t experts_per_launch) {
  (void)D;
  if (V <= 0 || N <= 0 || Dr <= 0 || !valid_dtype(dt)) return 0;
  const int64_t e = (experts_per_launch <= 0 || experts_per_launch > N) ? N : experts_per_launch;
  return (size_t)V * (size_t)Dr * dtype_size(dt) * (size_t)e;
}

extern "C" mole_status mole_build_lut(const void* embed, const void* W1, const void* W2, int64_t V, int64_t D,
                                      int32_t N, int64_t Dr, mole_act act, mole_dtype dt, void* lut,
                                      void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!valid_dtype(dt) || !valid_act(act)) return MOLE_ERR_ARG;
  if (V <= 0 || D <= 0 || N <= 0 || Dr <= 0) return MOLE_ERR_ARG;
  if (!embed || !W1 || !W2 || !lut) return MOLE_ERR_ARG;
  if (V > INT32_MAX || D > INT32_MAX || Dr > INT32_MAX) return MOLE_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < mole_build_lut_workspace(V, D, N, Dr, dt, 1)) return MOLE_ERR_WORKSPACE;
  mole_status st = check_device();
  if (st != MOLE_OK) return st;
  if (dt == MOLE_BF16 && mole::build_tc_supported(V, D, Dr, embed, W1, W2, lut, workspace))
    return mole::build_tc(embed, W1, W2, V, D, N, Dr, (int)act, lut, workspace, ws_bytes, stream);
  return mole::build_simt(embed, W1, W2, V, D, N, Dr, (int)act, dt == MOLE_BF16, lut, workspace, ws_bytes,
                          stream);
}

extern "C" mole_status mole_lookup_combine(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                           const void* lut, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                                           float* out, cudaStream_t stream) {
  if (!valid_dtype(dt)) return MOLE_ERR_ARG;
  mole_status st = check_combine(ids, T, h, Wr, lut, V, N, D, out);
  if (st != MOLE_OK) return st;
  if (dt == MOLE_BF16 && D % 16 != 0) return MOLE_ERR_UNSUPPORTED;
  if (dt == MOLE_F32 && D % 4 != 0) return MOLE_ERR_UNSUPPORTED;
  if (!mole::aligned16(lut)) return MOLE_ERR_ALIGN;
  if (T == 0) return MOLE_OK;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::combine_dispatch(ids, T, h, Wr, lut, nullptr, V, N, (int)D, dt == MOLE_BF16,
                                dt == MOLE_BF16 ? 0 : 1, out, stream);
}

extern "C" size_t mole_token_groups_workspace(int64_t T, int32_t N) { return mole::token_groups_bytes(T, N); }

extern "C" size_t mole_lookup_combine_grouped_workspace(int64_t T, int32_t N) {
  return mole::token_groups_bytes(T, N);
}

namespace {
mole_status check_groups(int64_t T, int32_t N, const void* groups, size_t bytes) {
  if (T == 0) return MOLE_OK;
  if (!groups || bytes < mole::token_groups_bytes(T, N)) return MOLE_ERR_WORKSPACE;
  if (!mole::aligned16(groups)) return MOLE_ERR_ALIGN;
  return MOLE_OK;
}

mole_status check_combine_bf16(const int32_t* ids, int64_t T, const void* h, const void* Wr, const void* lut,
                               int64_t V, int32_t N, int64_t D, mole_dtype dt, float* out) {
  if (!valid_dtype(dt)) return MOLE_ERR_ARG;
  mole_status st = check_combine(ids, T, h, Wr, lut, V, N, D, out);
  if (st != MOLE_OK) return st;
  if (dt == MOLE_BF16 && D % 16 != 0) return MOLE_ERR_UNSUPPORTED;
  if (dt == MOLE_F32 && D % 4 != 0) return MOLE_ERR_UNSUPPORTED;
  if (!mole::aligned16(lut)) return MOLE_ERR_ALIGN;
  return MOLE_OK;
}
}  // namespace

extern "C" mole_status mole_token_groups_build(const int32_t* ids, int64_t T, int64_t V, int32_t N, void* groups,
                                               size_t bytes, cudaStream_t stream) {
  if (T < 0 || V <= 0 || V > INT32_MAX || N <= 0) return MOLE_ERR_ARG;
  if (T > 0 && !ids) return MOLE_ERR_ARG;
  if (N > 32) return MOLE_ERR_UNSUPPORTED;
  mole_status st = check_groups(T, N, groups, bytes);
  if (st != MOLE_OK || T == 0) return st;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::token_groups_build(ids, T, V, N, groups, bytes, stream);
}

extern "C" mole_status mole_lookup_combine_groups(const int32_t* ids, int64_t T, const void* groups, size_t bytes,
                                                  const void* h, const void* Wr, const void* lut, int64_t V,
                                                  int32_t N, int64_t D, mole_dtype dt, float* out,
                                                  cudaStream_t stream) {
  mole_status st = check_combine_bf16(ids, T, h, Wr, lut, V, N, D, dt, out);
  if (st != MOLE_OK) return st;
  st = check_groups(T, N, groups, bytes);
  if (st != MOLE_OK || T == 0) return st;
  st = check_device();
  if (st != MOLE_OK) return st;
  if (dt == MOLE_BF16 && mole::aligned16(Wr)) {
    st = mole::combine_groups(groups, bytes, T, h, Wr, lut, nullptr, false, N, (int)D, out, stream);
    if (st != MOLE_ERR_UNSUPPORTED) return st;
  }
  return mole::combine_dispatch(ids, T, h, Wr, lut, nullptr, V, N, (int)D, dt == MOLE_BF16, dt == MOLE_BF16 ? 0 : 1,
                                out, stream);
}

extern "C" mole_status mole_lookup_combine_nf3_groups(const int32_t* ids, int64_t T, const void* groups,
                                                      size_t bytes, const void* h, const void* Wr,
                                                      const uint8_t* codes, const uint16_t* scales, int64_t V,
                                                      int32_t N, int64_t D, mole_dtype dt, float* out,
                                                      cudaStream_t stream) {
  if (!valid_dtype(dt)) return MOLE_ERR_ARG;
  mole_status st = check_combine(ids, T, h, Wr, codes, V, N, D, out);
  if (st != MOLE_OK) return st;
  if (T > 0 && !scales) return MOLE_ERR_ARG;
  if (D % 64 != 0) return MOLE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(scales) & 1u)) return MOLE_ERR_ALIGN;
  st = check_groups(T, N, groups, bytes);
  if (st != MOLE_OK || T == 0) return st;
  st = check_device();
  if (st != MOLE_OK) return st;
  if (dt == MOLE_BF16 && mole::aligned16(Wr) && mole::aligned16(codes) && mole::aligned16(scales)) {
    st = mole::combine_groups(groups, bytes, T, h, Wr, codes, scales, true, N, (int)D, out, stream);
    if (st != MOLE_ERR_UNSUPPORTED) return st;
  }
  return mole::combine_dispatch(ids, T, h, Wr, codes, scales, V, N, (int)D, dt == MOLE_BF16, 2, out, stream);
}

extern "C" mole_status mole_lookup_combine_grouped(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                                   const void* lut, int64_t V, int32_t N, int64_t D,
                                                   mole_dtype dt, float* out, void* workspace, size_t ws_bytes,
                                                   cudaStream_t stream) {
  mole_status st = check_combine_bf16(ids, T, h, Wr, lut, V, N, D, dt, out);
  if (st != MOLE_OK) return st;
  st = check_groups(T, N, workspace, ws_bytes);
  if (st != MOLE_OK || T == 0) return st;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::combine_grouped_dispatch(ids, T, h, Wr, lut, nullptr, V, N, (int)D, dt == MOLE_BF16,
                                        dt == MOLE_BF16 ? 0 : 1, out, workspace, ws_bytes, stream);
}

extern "C" mole_status mole_quantize_lut_nf3(const void* lut_bf16, int64_t V, int32_t N, int64_t D,
                                             uint8_t* codes, uint16_t* scales, cudaStream_t stream) {
  if (!lut_bf16 || !codes || !scales || V <= 0 || N <= 0 || D <= 0) return MOLE_ERR_ARG;
  if (D % 64 != 0) return MOLE_ERR_UNSUPPORTED;
  if (!mole::aligned16(lut_bf16) || !mole::aligned8(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return MOLE_ERR_ALIGN;
  mole_status st = check_device();
  if (st != MOLE_OK) return st;
  return mole::nf3_quantize_launch(lut_bf16, V, N, D, codes, scales, stream);
}

extern "C" mole_status mole_lookup_combine_nf3(const int32_t* ids, int64_t T, const void* h, const void* Wr,
                                               const uint8_t* codes, const uint16_t* scales, int64_t V,
                                               int32_t N, int64_t D, mole_dtype dt, float* out,
                                               cudaStream_t stream) {
  if (!valid_dtype(dt)) return MOLE_ERR_ARG;
  mole_status st = check_combine(ids, T, h, Wr, codes, V, N, D, out);
  if (st != MOLE_OK) return st;
  if (T > 0 && !scales) return MOLE_ERR_ARG;
  if (D % 64 != 0) return MOLE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return MOLE_ERR_ALIGN;
  if (T == 0) return MOLE_OK;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::combine_dispatch(ids, T, h, Wr, codes, scales, V, N, (int)D, dt == MOLE_BF16, 2, out, stream);
}

extern "C" void mole_nf3_levels(uint16_t levels_f16[8]) {
  float mid[7];
  mole::nf3_tables(levels_f16, mid);
}

extern "C" void mole_nf3_midpoints(float mid[7]) {
  uint16_t levels[8];
  mole::nf3_tables(levels, mid);
}

extern "C" mole_status mole_gather_plan(const int32_t* ids, int64_t T, int64_t V, int32_t* uniq,
                                        int32_t* n_uniq, int32_t* slot, cudaStream_t stream) {
  if (T < 0 || V <= 0 || !n_uniq) return MOLE_ERR_ARG;
  if (T > 0 && (!ids || !uniq || !slot)) return MOLE_ERR_ARG;
  if (T > INT32_MAX) return MOLE_ERR_UNSUPPORTED;
  mole_status st = check_device();
  if (st != MOLE_OK) return st;
  return mole::gather_plan_launch(ids, T, V, uniq, n_uniq, slot, stream);
}

namespace {
// Shared checks of the offloaded-table entry points.
mole_status check_offload(int64_t T, const void* groups, size_t bytes, int64_t V, int32_t N, int64_t D,
                          mole_dtype dt, int32_t nf3, const void* staging, size_t staging_bytes) {
  if (!valid_dtype(dt) || (nf3 != 0 && nf3 != 1)) return MOLE_ERR_ARG;
  if (T < 0 || V <= 0 || V > INT32_MAX || N <= 0 || D <= 0 || D > (1 << 20)) return MOLE_ERR_ARG;
  if (N > 32 || T > mole::kMaxOffloadT) return MOLE_ERR_UNSUPPORTED;
  if (nf3 ? D % 64 != 0 : (dt == MOLE_BF16 ? D % 16 != 0 : D % 4 != 0)) return MOLE_ERR_UNSUPPORTED;
  mole_status st = check_groups(T, N, groups, bytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!staging || staging_bytes < mole::offload_staging_bytes(T, V, N, (int)D, (int)dtype_size(dt), nf3 != 0))
    return MOLE_ERR_WORKSPACE;
  if (!mole::aligned16(staging)) return MOLE_ERR_ALIGN;
  return MOLE_OK;
}
}  // namespace

extern "C" size_t mole_offload_staging_bytes(int64_t T, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                                             int32_t nf3) {
  if (T <= 0 || V <= 0 || N <= 0 || N > 32 || D <= 0 || !valid_dtype(dt) || (nf3 != 0 && nf3 != 1)) return 0;
  if (nf3 && D % 64 != 0) return 0;
  return mole::offload_staging_bytes(T, V, N, (int)D, (int)dtype_size(dt), nf3 != 0);
}

extern "C" mole_status mole_offload_stage(int64_t T, const void* groups, size_t bytes, const void* table,
                                          const uint16_t* scales, int64_t V, int32_t N, int64_t D, mole_dtype dt,
                                          int32_t nf3, void* staging, size_t staging_bytes, int32_t* n_rows,
                                          cudaStream_t stream) {
  mole_status st = check_offload(T, groups, bytes, V, N, D, dt, nf3, staging, staging_bytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!table || (nf3 && !scales)) return MOLE_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(n_rows) & 3u) return MOLE_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(table) & (nf3 ? 7u : 15u)) || (nf3 && (reinterpret_cast<uintptr_t>(scales) & 1u)))
    return MOLE_ERR_ALIGN;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::offload_stage(groups, bytes, T, table, scales, V, N, (int)D, (int)dtype_size(dt), nf3 != 0, staging,
                             staging_bytes, n_rows, stream);
}

extern "C" mole_status mole_lookup_combine_offload(int64_t T, const void* groups, size_t bytes, const void* h,
                                                   const void* Wr, const void* staging, size_t staging_bytes,
                                                   int64_t V, int32_t N, int64_t D, mole_dtype dt, int32_t nf3,
                                                   float* out, cudaStream_t stream) {
  mole_status st = check_offload(T, groups, bytes, V, N, D, dt, nf3, staging, staging_bytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!h || !Wr || !out) return MOLE_ERR_ARG;
  if (!mole::aligned16(h) || !mole::aligned16(out)) return MOLE_ERR_ALIGN;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::combine_offload(groups, bytes, T, h, Wr, staging, staging_bytes, V, N, (int)D, dt == MOLE_BF16,
                               nf3 != 0, out, stream);
}

extern "C" size_t mole_shared_ffn_workspace(int64_t T, int64_t Ds) {
  if (T <= 0 || Ds <= 0) return 0;
  return (size_t)T * (size_t)Ds * 2;
}

extern "C" mole_status mole_shared_ffn(const void* h, const void* W1s, const void* W2s, int64_t T, int64_t D,
                                       int64_t Ds, mole_act act, const float* add, const float* residual, float* out,
                                       void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!valid_act(act) || T < 0 || D <= 0 || Ds <= 0) return MOLE_ERR_ARG;
  if (T == 0) return MOLE_OK;
  if (!h || !W1s || !W2s || !out) return MOLE_ERR_ARG;
  if (D % 64 != 0 || Ds % 64 != 0 || T > INT32_MAX || D > INT32_MAX || Ds > INT32_MAX) return MOLE_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < mole_shared_ffn_workspace(T, Ds)) return MOLE_ERR_WORKSPACE;
  if (!mole::aligned16(h) || !mole::aligned16(W1s) || !mole::aligned16(W2s) || !mole::aligned16(add) ||
      !mole::aligned16(residual) || !mole::aligned16(out) || !mole::aligned16(workspace))
    return MOLE_ERR_ALIGN;
  mole_status st = check_device();
  if (st != MOLE_OK) return st;
  if (!mole::shared_ffn_tc_supported(T, D, Ds, h, W1s, W2s, add, residual, out, workspace))
    return MOLE_ERR_UNSUPPORTED;
  return mole::shared_ffn_tc(h, W1s, W2s, T, D, Ds, (int)act, add, residual, out, workspace, ws_bytes, stream);
}

extern "C" size_t mole_ffn_block_workspace(int64_t T, int64_t D, int64_t Ds) {
  if (T <= 0 || D <= 0 || Ds <= 0) return 0;
  const size_t h_bytes = ((size_t)T * (size_t)Ds * 2 + 255) / 256 * 256;
  return h_bytes + (size_t)T * (size_t)D * 4;
}

extern "C" mole_status mole_ffn_block(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes,
                                      const void* h, const void* Wr, const void* lut, int64_t V, int32_t N,
                                      const void* W1s, const void* W2s, int64_t D, int64_t Ds, mole_act act,
                                      const float* residual, float* out, void* workspace, size_t ws_bytes,
                                      cudaStream_t stream) {
  if (!valid_act(act)) return MOLE_ERR_ARG;
  mole_status st = check_combine_bf16(ids, T, h, Wr, lut, V, N, D, MOLE_BF16, out);
  if (st != MOLE_OK) return st;
  st = check_groups(T, N, groups, groups_bytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!W1s || !W2s || Ds <= 0) return MOLE_ERR_ARG;
  if (D % 64 != 0 || Ds % 64 != 0 || T > INT32_MAX || Ds > INT32_MAX) return MOLE_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < mole_ffn_block_workspace(T, D, Ds)) return MOLE_ERR_WORKSPACE;
  if (!mole::aligned16(W1s) || !mole::aligned16(W2s) || !mole::aligned16(residual) || !mole::aligned16(workspace))
    return MOLE_ERR_ALIGN;
  st = check_device();
  if (st != MOLE_OK) return st;
  // the routed-expert mixture into the workspace (fp32 [T, D]), then the
  // shared expert with the mixture and the residual added in its epilogue
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t h_bytes = ((size_t)T * (size_t)Ds * 2 + 255) / 256 * 256;
  float* mix = reinterpret_cast<float*>(ws + h_bytes);
  if (!mole::shared_ffn_tc_supported(T, D, Ds, h, W1s, W2s, mix, residual, out, ws)) return MOLE_ERR_UNSUPPORTED;
  st = mole_lookup_combine_groups(ids, T, groups, groups_bytes, h, Wr, lut, V, N, D, MOLE_BF16, mix, stream);
  if (st != MOLE_OK) return st;
  return mole::shared_ffn_tc(h, W1s, W2s, T, D, Ds, (int)act, mix, residual, out, ws, h_bytes, stream);
}

extern "C" mole_status mole_build_lut_nf3(const void* embed, const void* W1, const void* W2, int64_t V, int64_t D,
                                          int32_t N, int64_t Dr, mole_act act, uint8_t* codes, uint16_t* scales,
                                          void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!valid_act(act)) return MOLE_ERR_ARG;
  if (V <= 0 || D <= 0 || N <= 0 || Dr <= 0) return MOLE_ERR_ARG;
  if (!embed || !W1 || !W2 || !codes || !scales) return MOLE_ERR_ARG;
  if (V > INT32_MAX || D > INT32_MAX || Dr > INT32_MAX || D % 64 != 0 || Dr % 64 != 0) return MOLE_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < mole_build_lut_workspace(V, D, N, Dr, MOLE_BF16, 1)) return MOLE_ERR_WORKSPACE;
  if (!mole::aligned8(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u)) return MOLE_ERR_ALIGN;
  mole_status st = check_device();
  if (st != MOLE_OK) return st;
  if (!mole::build_tc_supported(V, D, Dr, embed, W1, W2, workspace, workspace)) return MOLE_ERR_UNSUPPORTED;
  return mole::build_tc_nf3(embed, W1, W2, V, D, N, Dr, (int)act, codes, scales, workspace, ws_bytes, stream);
}

extern "C" size_t mole_train_cache_bytes(int64_t T, int64_t V, int32_t N, int64_t D, int64_t Dr) {
  if (T <= 0 || V <= 0 || N <= 0 || N > 32 || D <= 0 || Dr <= 0) return 0;
  return mole::train_cache_bytes(T, V, N, D, Dr);
}

namespace {
mole_status check_train(int64_t T, const void* groups, size_t gbytes, const void* h, const void* Wr, const void* W1,
                        const void* W2, int64_t V, int32_t N, int64_t D, int64_t Dr, mole_act act, const void* cache,
                        size_t cbytes) {
  if (!valid_act(act) || T < 0 || V <= 0 || V > INT32_MAX || N <= 0 || D <= 0 || Dr <= 0) return MOLE_ERR_ARG;
  if (T > 0 && (!h || !Wr || !W1 || !W2)) return MOLE_ERR_ARG;
  if (N > 32 || D % 64 != 0 || Dr % 64 != 0 || T > INT32_MAX || D > INT32_MAX || Dr > INT32_MAX)
    return MOLE_ERR_UNSUPPORTED;
  mole_status st = check_groups(T, N, groups, gbytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!cache || cbytes < mole::train_cache_bytes(T, V, N, D, Dr)) return MOLE_ERR_WORKSPACE;
  if (!mole::aligned16(h) || !mole::aligned16(Wr) || !mole::aligned16(W1) || !mole::aligned16(W2) ||
      !mole::aligned16(cache))
    return MOLE_ERR_ALIGN;
  return MOLE_OK;
}
}  // namespace

extern "C" mole_status mole_train_forward(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes,
                                          const void* h, const void* Wr, const void* E, const void* W1,
                                          const void* W2, int64_t V, int32_t N, int64_t D, int64_t Dr, mole_act act,
                                          float* out, void* cache, size_t cache_bytes, int32_t* n_distinct,
                                          cudaStream_t stream) {
  mole_status st = check_train(T, groups, groups_bytes, h, Wr, W1, W2, V, N, D, Dr, act, cache, cache_bytes);
  if (st != MOLE_OK) return st;
  if (n_distinct) *n_distinct = 0;
  if (T == 0) return MOLE_OK;
  if (!ids || !E || !out || !n_distinct) return MOLE_ERR_ARG;
  if (!mole::aligned16(E) || !mole::aligned16(out)) return MOLE_ERR_ALIGN;
  st = check_device();
  if (st != MOLE_OK) return st;
  if (!mole::build_tc_supported(std::min(T, V), D, Dr, E, W1, W2, cache, cache)) return MOLE_ERR_UNSUPPORTED;
  return mole::train_forward(groups, groups_bytes, T, h, Wr, E, W1, W2, V, N, D, Dr, (int)act, out, cache,
                             cache_bytes, n_distinct, stream);
}

extern "C" mole_status mole_train_backward(const int32_t* ids, int64_t T, const void* groups, size_t groups_bytes,
                                           const void* h, const void* Wr, const void* E, const void* W1,
                                           const void* W2, int64_t V, int32_t N, int64_t D, int64_t Dr, mole_act act,
                                           const float* dout, void* cache, size_t cache_bytes, int32_t n_distinct,
                                           float* dh, float* dWr, float* dE, float* dW1, float* dW2,
                                           cudaStream_t stream) {
  (void)ids;
  (void)E;
  mole_status st = check_train(T, groups, groups_bytes, h, Wr, W1, W2, V, N, D, Dr, act, cache, cache_bytes);
  if (st != MOLE_OK || T == 0) return st;
  if (!dout) return MOLE_ERR_ARG;
  if (n_distinct < 0 || n_distinct > std::min(T, V)) return MOLE_ERR_ARG;
  st = check_device();
  if (st != MOLE_OK) return st;
  return mole::train_backward(groups, groups_bytes, T, h, Wr, W1, W2, V, N, D, Dr, (int)act, dout, cache, cache_bytes,
                              n_distinct, dh, dWr, dE, dW1, dW2, stream);
}
