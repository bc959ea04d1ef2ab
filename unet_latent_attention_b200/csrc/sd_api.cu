// Library-wide entry points: status strings, per-thread error text, the device status word.
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "sd_internal.h"

namespace {

thread_local char g_last_error[512] = "";

// One status word per device (a __device__ variable exists once per device that loads the module).
__device__ unsigned int g_status_word = 0;

constexpr int kMaxDevices = 64;
unsigned int* g_status_addr[kMaxDevices] = {};
void* g_status_ctx[kMaxDevices] = {};  // the context each cached address was resolved in
int g_sm_count[kMaxDevices] = {};
std::mutex g_mu;

}  // namespace

namespace sd {

sd_status fail(sd_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

sd_status cuda_check(cudaError_t err, const char* where) {
  if (err == cudaSuccess) return SD_OK;
  return fail(SD_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(err), cudaGetErrorString(err));
}

sd_status current_context(void** ctx) {
  using GetCurrent = int (*)(void**);  // cuCtxGetCurrent(CUcontext*): CUresult
  static GetCurrent fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrent>(p);
  });
  if (!fn) return fail(SD_ERR_CUDA, "cuCtxGetCurrent is unavailable");
  *ctx = nullptr;
  if (fn(ctx) != 0) return fail(SD_ERR_CUDA, "cuCtxGetCurrent failed");
  return SD_OK;
}

unsigned int* device_status_word() {
  int dev = 0;
  if (cuda_check(cudaGetDevice(&dev), "cudaGetDevice") != SD_OK || dev >= kMaxDevices) return nullptr;
  // cudaGetDevice makes the primary context current if none is; the address belongs to it.
  void* ctx = nullptr;
  if (current_context(&ctx) != SD_OK) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_addr[dev] || g_status_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cuda_check(cudaGetSymbolAddress(&p, g_status_word), "cudaGetSymbolAddress(status)") != SD_OK)
      return nullptr;
    g_status_addr[dev] = static_cast<unsigned int*>(p);
    g_status_ctx[dev] = ctx;
  }
  return g_status_addr[dev];
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

}  // namespace sd

extern "C" {

const char* sd_status_string(sd_status status) {
  switch (status) {
    case SD_OK: return "SD_OK";
    case SD_ERR_INVALID_ARG: return "SD_ERR_INVALID_ARG";
    case SD_ERR_UNSUPPORTED: return "SD_ERR_UNSUPPORTED";
    case SD_ERR_MISALIGNED: return "SD_ERR_MISALIGNED";
    case SD_ERR_CUDA: return "SD_ERR_CUDA";
    case SD_ERR_TIMEOUT: return "SD_ERR_TIMEOUT";
  }
  return "SD_ERR_UNKNOWN";
}

const char* sd_last_error(void) { return g_last_error; }

sd_status sd_device_status(void* stream, int reset) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int* word = sd::device_status_word();
  if (!word) return SD_ERR_CUDA;
  unsigned int host = 0;
  sd_status st = sd::cuda_check(cudaMemcpyAsync(&host, word, sizeof(host), cudaMemcpyDeviceToHost, s),
                                "cudaMemcpyAsync(status)");
  if (st == SD_OK) st = sd::cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st != SD_OK) return st;
  if (reset) {
    st = sd::cuda_check(cudaMemsetAsync(word, 0, sizeof(unsigned int), s), "cudaMemsetAsync(status)");
    // An aborted attention launch may have left hand-off flags set: clear them with the word.
    if (st == SD_OK && host != 0) st = sd::attention_clear_handoff(s);
    if (st == SD_OK) st = sd::cuda_check(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    if (st != SD_OK) return st;
  }
  if (host & sd::kDevErrTimeout)
    return sd::fail(SD_ERR_TIMEOUT, "a kernel gave up a bounded wait (status word 0x%x)", host);
  return SD_OK;
}

int sd_version(void) { return 100; }

}  // extern "C"
