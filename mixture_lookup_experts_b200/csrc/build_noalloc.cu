// build_noalloc.cu -- table build for callers that cannot allocate device memory.
//
// mole_build_lut needs a scratch buffer for the expert hidden activations, and
// the caller usually allocates it.  Some callers cannot: serving loops that
// forbid device allocations after start-up so that their memory use stays
// fixed, and plugin hosts that hand out all device memory through their own
// pool and give plugins no allocator.  For them, mole_build_lut_noalloc runs
// the same build kernels with the scratch taken from a fixed array in this
// library's device memory (16 MiB; every GPU that loads the library holds it
// until the process exits).
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;

// The scratch array.  Host code must not pass its name to a kernel (on the
// host it is only a stand-in symbol); scratch_device_ptr() resolves the device
// address once per device (and context).
static __device__ __align__(256) uint8_t g_build_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchAddr {
  unsigned long long ctx_id;  // the context the address belongs to
  void* ptr;
};
ScratchAddr g_scratch[kMaxDevices];

typedef CUresult (*ctx_get_current_t)(CUcontext*);
typedef CUresult (*ctx_get_id_t)(CUcontext, unsigned long long*);

// Unique id of the current context (cuCtxGetId, fetched from the driver at
// run time); 0 if it cannot be read.  A device reset or a new primary
// context gets a new id, and with it the array a new device address.
unsigned long long current_context_id() {
  static ctx_get_current_t get_current = nullptr;
  static ctx_get_id_t get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<ctx_get_current_t>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<ctx_get_id_t>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_build_scratch on the current device: looked up
// (cudaGetSymbolAddress, with the device current) on the first call per
// device, and again only when the device's context has changed since (after a
// device reset the module is loaded anew and the array moves).  nullptr if the
// lookup fails.
void* scratch_device_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& s = g_scratch[dev];
  if (s.ptr && s.ctx_id != 0 && s.ctx_id == current_context_id()) return s.ptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_build_scratch) != cudaSuccess || !p) return nullptr;
  s = ScratchAddr{current_context_id(), p};  // the lookup has made the context current
  return s.ptr;
}

}  // namespace

extern "C" mole_status mole_build_lut_noalloc(const void* embed, const void* W1, const void* W2, int64_t V,
                                              int64_t D, int32_t N, int64_t Dr, mole_act act, mole_dtype dt,
                                              void* lut, cudaStream_t stream) {
  if (dt != MOLE_F32 && dt != MOLE_BF16) return MOLE_ERR_ARG;
  if (act < MOLE_ACT_GELU_ERF || act > MOLE_ACT_IDENTITY) return MOLE_ERR_ARG;
  if (V <= 0 || D <= 0 || N <= 0 || Dr <= 0) return MOLE_ERR_ARG;
  if (!embed || !W1 || !W2 || !lut) return MOLE_ERR_ARG;
  if (V > INT32_MAX || D > INT32_MAX || Dr > INT32_MAX) return MOLE_ERR_UNSUPPORTED;
  // One expert's hidden activations must fit in the fixed scratch.
  const size_t per_expert = (size_t)V * (size_t)Dr * (dt == MOLE_BF16 ? 2u : 4u);
  if (per_expert > kScratchBytes) return MOLE_ERR_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return MOLE_ERR_NO_DEVICE;
  void* ws = scratch_device_ptr();
  if (!ws) return MOLE_ERR_CUDA;
  if (dt == MOLE_BF16 && mole::build_tc_supported(V, D, Dr, embed, W1, W2, lut, ws))
    return mole::build_tc(embed, W1, W2, V, D, N, Dr, (int)act, lut, ws, kScratchBytes, stream);
  return mole::build_simt(embed, W1, W2, V, D, N, Dr, (int)act, dt == MOLE_BF16, lut, ws, kScratchBytes, stream);
}
