// Status word, error messages, workspace sizes and the small support calls of
// the C ABI (see include/tps.h).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "tps_internal.cuh"

namespace tps {

static thread_local char g_msg[512] = {0};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_msg[0] = 0;
  return TPS_OK;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TPS_OK;
  return fail(TPS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Host-side fault injection for tests: the next n launch checks report a launch
// failure (after consuming the real launch status) instead of success.
static std::atomic<int> g_inject_launch_failures{0};

int launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  int n = g_inject_launch_failures.load();
  while (n > 0 && !g_inject_launch_failures.compare_exchange_weak(n, n - 1)) {
  }
  if (n > 0) return fail(TPS_ERR_CUDA, "%s: injected launch failure (test hook)", what);
  return cuda_status(e, what);
}

// One status word per device: bit 0 = an out-of-range index was skipped,
// bit 1 = a bounded wait gave up.
static __device__ unsigned int g_status_word;

static constexpr int kMaxDevices = 64;
static unsigned int* g_status_ptr[kMaxDevices];
static int g_sms[kMaxDevices];
static std::mutex g_mu;

unsigned int* device_status(int* err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = cuda_status(e == cudaSuccess ? cudaErrorInvalidDevice : e, "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) {
      *err = cuda_status(e, "cudaGetSymbolAddress(status)");
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *err = TPS_OK;
  return g_status_ptr[dev];
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

}  // namespace tps

extern "C" {

const char* tps_last_error(void) { return tps::g_msg; }

void tps_debug_inject_launch_failures(int n) { tps::g_inject_launch_failures.store(n > 0 ? n : 0); }

int tps_pointer_is_device_accessible(const void* p) {
  if (!p) return 0;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();   // clear the (non-sticky) error an unknown pointer leaves behind
    return 0;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      return 1;
    case cudaMemoryTypeHost:
      return a.devicePointer == p ? 1 : 0;
    default:
      return 0;
  }
}

const char* tps_version(void) { return "libtps 0.1.0 (sm_100a)"; }

int tps_check(tps_stream stream) {
  int err = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return tps::cuda_status(e, "cudaStreamSynchronize");
  unsigned int* st = tps::device_status(&err);
  if (!st) return err;
  unsigned int v = 0;
  e = cudaMemcpy(&v, st, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return tps::cuda_status(e, "read status word");
  if (v) {
    unsigned int zero = 0;
    e = cudaMemcpy(st, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return tps::cuda_status(e, "clear status word");
  }
  if (v & tps::STATUS_TIMEOUT) return tps::fail(TPS_ERR_TIMEOUT, "a bounded device wait gave up");
  if (v & tps::STATUS_BOUNDS) return tps::fail(TPS_ERR_BOUNDS, "an index outside [0, N) was skipped");
  return tps::ok();
}

}  // extern "C"
