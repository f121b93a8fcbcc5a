// status.cu -- per-device error word, device queries, mole_check / mole_status_str.
#include <chrono>
#include <mutex>
#include <thread>

#include "common.cuh"

namespace mole {

// One error word per device (a static device variable: no allocation).
__device__ unsigned g_error_word;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];
}  // namespace

unsigned* error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  return g_err_ptr[dev];
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

}  // namespace mole

extern "C" const char* mole_status_str(mole_status s) {
  switch (s) {
    case MOLE_OK: return "ok";
    case MOLE_ERR_ARG: return "invalid argument";
    case MOLE_ERR_ALIGN: return "misaligned pointer";
    case MOLE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOLE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOLE_ERR_INDEX: return "token id out of range";
    case MOLE_ERR_CUDA: return "CUDA error";
    case MOLE_ERR_TIMEOUT: return "timed out";
    case MOLE_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

extern "C" int mole_version(void) { return 100; }

extern "C" mole_status mole_check(cudaStream_t stream, int timeout_ms) {
  if (timeout_ms < 0) return MOLE_ERR_ARG;  // every host wait has a limit
  using clock = std::chrono::steady_clock;
  const auto t0 = clock::now();
  for (;;) {
    cudaError_t e = cudaStreamQuery(stream);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return MOLE_ERR_CUDA;
    if (std::chrono::duration_cast<std::chrono::milliseconds>(clock::now() - t0).count() > timeout_ms)
      return MOLE_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
  unsigned* w = mole::error_word();
  if (!w) return MOLE_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, w, sizeof v, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return MOLE_ERR_CUDA;
  if (cudaMemsetAsync(w, 0, sizeof v, stream) != cudaSuccess) return MOLE_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOLE_ERR_CUDA;
  if (v & mole::kErrTimeout) return MOLE_ERR_TIMEOUT;
  if (v & mole::kErrIndex) return MOLE_ERR_INDEX;
  if (v & mole::kErrGrouping) return MOLE_ERR_ARG;
  return MOLE_OK;
}
