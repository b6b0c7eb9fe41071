// api.cu -- error reporting, the device status word, and the bounded-wait
// self test.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <set>
#include <utility>

#include "frt_common.cuh"
#include "frt_sm100.cuh"

namespace frt {

static thread_local char g_err[512] = {0};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = 0; }

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(FRT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return FRT_OK;
}

// One status word per device: bounded waits that run out store FRT_ETIMEOUT.
__device__ int g_status_word;

static constexpr int kMaxDevices = 64;
static int* g_status_ptr[kMaxDevices] = {nullptr};
static int g_sms[kMaxDevices] = {0};

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return 148;
  if (!g_sms[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = n > 0 ? n : 148;
  }
  return g_sms[dev];
}

bool first_use(const void* kernel) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> seen;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  return seen.insert({dev, kernel}).second;
}

// A single CTA waits on an mbarrier whose arrival count is never reached.
__global__ void bounded_wait_probe(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = mbar_wait_bounded(&bar, 0, timeout_ns, nullptr);
    if (!ok) atomicExch(status, FRT_ETIMEOUT);
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace frt

extern "C" const char* frt_last_error(void) { return frt::g_err; }

extern "C" int frt_version(void) { return 100; }

extern "C" int frt_device_status(int reset, void* stream) {
  frt::clear_error();
  int* p = frt::device_status_ptr();
  if (!p) return frt::fail(FRT_ECUDA, "device status word unavailable");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, p, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return frt::fail(FRT_ECUDA, "reading the device status word: %s",
                     cudaGetErrorString(cudaGetLastError()));
  if (reset) {
    if (cudaMemsetAsync(p, 0, sizeof(int), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return frt::fail(FRT_ECUDA, "clearing the device status word");
  }
  if (h == FRT_ETIMEOUT)
    return frt::fail(FRT_ETIMEOUT, "a bounded device wait ran out");
  return h == 0 ? FRT_OK : frt::fail(FRT_ECUDA, "device status %d", h);
}

extern "C" int frt_selftest_bounded_wait(int timeout_us, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(timeout_us > 0 && timeout_us <= 2000000, FRT_EINVAL,
              "timeout_us must be in (0, 2e6], got %d", timeout_us);
  int* st = frt::device_status_ptr();
  FRT_REQUIRE(st, FRT_ECUDA, "device status word unavailable");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(st, 0, sizeof(int), s) != cudaSuccess)
    return frt::fail(FRT_ECUDA, "clearing the device status word");
  frt::bounded_wait_probe<<<1, 32, 0, s>>>(st, uint64_t(timeout_us) * 1000ull);
  int rc = frt::check_launch("bounded_wait_probe");
  if (rc) return rc;
  return frt_device_status(1, stream);
}
