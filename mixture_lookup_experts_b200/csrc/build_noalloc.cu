// build_noalloc.cu -- table build for callers that cannot allocate device memory.
//
// mole_build_lut needs a scratch buffer for the expert hidden activations, and
// the caller usually allocates it.  Some callers cannot: code that runs while a
// stream is being captured into a CUDA graph (an allocation there breaks or
// invalidates the capture), serving loops that forbid device allocations after
// start-up so their memory use stays fixed, and plugin hosts that hand out all
// device memory through their own pool and give plugins no allocator.  For
// them, mole_build_lut_noalloc runs the same build kernels with the scratch
// taken from a fixed array in this library's device memory (16 MiB; every GPU
// that loads the library holds it until the process exits).
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;

// The scratch array.  Host code must not pass its name to a kernel (on the
// host it is only a stand-in symbol); scratch_device_ptr() resolves the device
// address once per device.
static __device__ __align__(256) uint8_t g_build_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of g_build_scratch on the current device (set up on the
// first call per device; nullptr if the lookup fails).
void* scratch_device_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_build_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
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
