// Library-wide entry points: device error word, status strings, version.
#include <cstdio>
#include <mutex>

#include "pa_common.cuh"

namespace pa {

// One error word per device; kernels OR PA_DEVERR_* bits into it.
__device__ unsigned int g_error_word;

namespace {
constexpr int kMaxDevices = 64;
unsigned int* g_err_ptr[kMaxDevices] = {};
std::mutex g_err_mu;
}  // namespace

unsigned int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_err_ptr[dev];
}

namespace {
thread_local char g_last_error[256] = "";
}

int record_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
  return PA_ERR_CUDA;
}

}  // namespace pa

extern "C" PA_API const char* pa_last_cuda_error(void) { return pa::g_last_error; }

extern "C" PA_API int pa_read_error_flags(uint32_t* host_flags, int clear) {
  if (!host_flags) return PA_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_error_word, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  *host_flags = v;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

extern "C" PA_API const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_NULL: return "PA_ERR_NULL: a required pointer is NULL";
    case PA_ERR_SHAPE: return "PA_ERR_SHAPE: invalid or inconsistent size";
    case PA_ERR_DTYPE: return "PA_ERR_DTYPE: unsupported dtype for this entry point";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: head dim / block size / group size not supported";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: split-KV partition size or count invalid";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime or launch error";
    case PA_ERR_ALIGN: return "PA_ERR_ALIGN: pointer not 16-byte aligned";
    default: return "unknown pa_status";
  }
}

extern "C" PA_API int pa_version(void) { return 100; }

extern "C" PA_API int pa_splitkv_num_partitions(int max_context_len, int partition_size) {
  if (partition_size <= 0) return 0;
  if (max_context_len <= 0) return 1;
  return (max_context_len + partition_size - 1) / partition_size;
}
