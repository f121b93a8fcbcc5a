// prefetch.cu -- cross-layer row prefetch for a step.  MoLE page, 推理阶段 and
// 复杂度分析: every MoLE layer indexes its table with the step's input token
// ids, so a step knows the rows of all of its layers before the first layer
// runs.  mole_prefetch_rows asks the L2 cache for those rows up front (bulk
// L2 prefetches, no data moved to the SMs and no wait), so that each layer's
// combine finds its rows in L2 instead of paying the HBM latency in turn.
//
// Work item = (table, token); its row is split into pieces of kPiece bytes
// spread over the lanes of a warp; one warp per CTA so that the prefetches
// leave from many SMs' copy engines at once.
#include "common.cuh"

namespace mole {
namespace {

constexpr int kMaxTables = 64;
constexpr int64_t kPiece = 4096;

struct TableList {
  const uint8_t* base[kMaxTables];
};

__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__global__ void __launch_bounds__(32) prefetch_rows_kernel(const int32_t* __restrict__ ids, int64_t T, TableList tl,
                                                           int n_tables, int64_t V, int64_t row_bytes) {
  pdl_trigger();  // the next kernel may start now; it does not read what this one touches
  const int lane = threadIdx.x;
  const int64_t items = (int64_t)n_tables * T;
  const int64_t pieces = (row_bytes + kPiece - 1) / kPiece;
  for (int64_t i = blockIdx.x; i < items; i += gridDim.x) {
    const int l = (int)(i / T);
    const int64_t t = i - (int64_t)l * T;
    const int32_t id = __ldg(ids + t);
    if (id < 0 || (int64_t)id >= V) continue;  // the layer's combine reports it
    const uint8_t* row = tl.base[l] + (int64_t)id * row_bytes;
    for (int64_t q = lane; q < pieces; q += 32) {
      const int64_t off = q * kPiece;
      const int64_t n = row_bytes - off < kPiece ? row_bytes - off : kPiece;
      bulk_prefetch_l2(row + off, (uint32_t)n);
    }
  }
}

}  // namespace
}  // namespace mole

extern "C" mole_status mole_prefetch_rows(const int32_t* ids, int64_t T, const void* const* tables, int32_t n_tables,
                                          int64_t V, int64_t row_bytes, cudaStream_t stream) {
  using namespace mole;
  if (T < 0 || V <= 0 || n_tables < 0 || row_bytes <= 0 || (T > 0 && ids == nullptr) ||
      (n_tables > 0 && tables == nullptr))
    return MOLE_ERR_ARG;
  if (row_bytes % 16 != 0) return MOLE_ERR_ALIGN;
  if (n_tables > kMaxTables) return MOLE_ERR_UNSUPPORTED;
  TableList tl{};
  for (int l = 0; l < n_tables; ++l) {
    if (tables[l] == nullptr) return MOLE_ERR_ARG;
    if (!aligned16(tables[l])) return MOLE_ERR_ALIGN;
    tl.base[l] = static_cast<const uint8_t*>(tables[l]);
  }
  if (T == 0 || n_tables == 0) return MOLE_OK;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return MOLE_ERR_NO_DEVICE;
  const int n_sm = num_sms();
  if (n_sm <= 0) return MOLE_ERR_NO_DEVICE;
  const int64_t items = (int64_t)n_tables * T;
  const unsigned grid = (unsigned)std::min<int64_t>(items, (int64_t)n_sm * 8);
  return cuda_status(launch_pdl(prefetch_rows_kernel, grid, 32, 0, stream, ids, T, tl, (int)n_tables, V, row_bytes));
}
