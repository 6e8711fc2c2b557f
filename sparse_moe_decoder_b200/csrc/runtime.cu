// libzmoe runtime: version, status strings, thread-local last error, the device error
// counter and cached device properties.
#include <mutex>
#include <string>

#include "common.cuh"

namespace zmoe {

namespace {
thread_local std::string g_last_error;

// One error counter per device that loads this library.  Kernels receive its device
// address as an argument; host code never dereferences it.
__device__ unsigned int g_device_errors;
// One timeout counter per device: kernels with bounded waits count here when a wait gives up.
__device__ unsigned int g_device_timeouts;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned int* g_counter_addr[kMaxDevices] = {};
unsigned int* g_timeout_addr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
int g_smem_optin[kMaxDevices] = {};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}
}  // namespace

zmoe_status fail(zmoe_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

void clear_error() { g_last_error.clear(); }

zmoe_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return ZMOE_OK;
}

unsigned int* device_error_counter() {
  int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_counter_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_errors) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_counter_addr[dev] = static_cast<unsigned int*>(p);
  }
  return g_counter_addr[dev];
}

unsigned int* device_timeout_counter() {
  int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_timeout_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_timeouts) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_timeout_addr[dev] = static_cast<unsigned int*>(p);
  }
  return g_timeout_addr[dev];
}

int num_sms() {
  int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_sms[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    g_sms[dev] = v;
  }
  return g_sms[dev];
}

int max_smem_optin() {
  int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 227 * 1024;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_smem_optin[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 227 * 1024;
    }
    g_smem_optin[dev] = v;
  }
  return g_smem_optin[dev];
}

}  // namespace zmoe

extern "C" {

int zmoe_version(void) { return 100; }  // 0.1.0

const char* zmoe_status_string(int status) {
  switch (status) {
    case ZMOE_OK: return "ok";
    case ZMOE_ERR_INVALID_ARG: return "invalid argument";
    case ZMOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ZMOE_ERR_CUDA: return "CUDA error";
    case ZMOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case ZMOE_ERR_DEVICE_CHECK: return "device-side data check failed";
    case ZMOE_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

const char* zmoe_last_error(void) { return zmoe::g_last_error.c_str(); }

zmoe_status zmoe_get_device_errors(zmoe_stream_t stream, uint32_t* count) {
  if (!count) return zmoe::fail(ZMOE_ERR_INVALID_ARG, "zmoe_get_device_errors: count is NULL");
  *count = 0;
  unsigned int* err = zmoe::device_error_counter();
  unsigned int* tmo = zmoe::device_timeout_counter();
  if (!err || !tmo) return zmoe::fail(ZMOE_ERR_CUDA, "zmoe_get_device_errors: no device counters");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int host[2] = {0, 0};
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&host[0], err, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&host[1], tmo, sizeof(unsigned int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemset(tmo, 0, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return zmoe::fail(ZMOE_ERR_CUDA, std::string("zmoe_get_device_errors: ") + cudaGetErrorString(e));
  *count = host[0] + host[1];
  zmoe::clear_error();
  if (host[1]) return zmoe::fail(ZMOE_ERR_TIMEOUT, "a bounded device-side wait gave up");
  return host[0] ? ZMOE_ERR_DEVICE_CHECK : ZMOE_OK;
}

}  // extern "C"
