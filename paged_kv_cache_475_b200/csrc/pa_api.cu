// Library-wide entry points: device error word, workspace sizes, status strings, version.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "pa_common.cuh"

namespace pa {

// One error word per device; kernels OR PA_DEVERR_* bits into it.
__device__ unsigned int g_error_word;

uint64_t current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id);
}

namespace {
constexpr int kMaxDevices = 64;
ContextCached<unsigned int*> g_err_ptr[kMaxDevices];
std::mutex g_err_mu;
}  // namespace

unsigned int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev].valid()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev].set(static_cast<unsigned int*>(p));
  }
  return g_err_ptr[dev].value;
}

namespace {
thread_local char g_last_error[256] = "";
}

int record_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
  return PA_ERR_CUDA;
}

}  // namespace pa

namespace pa {
#if PA_TRACE
__device__ TraceRecord g_trace[kTraceMax];
#endif
TraceRecord* trace_buffer() {
#if PA_TRACE
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_trace) == cudaSuccess ? static_cast<TraceRecord*>(p) : nullptr;
#else
  return nullptr;
#endif
}
}  // namespace pa

extern "C" PA_API int pa_trace_read(void* host_records, int max_records) {
#if PA_TRACE
  if (!host_records || max_records <= 0) return PA_ERR_NULL;
  const int n = max_records < pa::kTraceMax ? max_records : pa::kTraceMax;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  const cudaError_t e = cudaMemcpyFromSymbol(host_records, pa::g_trace, sizeof(pa::TraceRecord) * n);
  if (e != cudaSuccess) return pa::record_cuda_error(e, "trace: copy the records");
  return PA_OK;
#else
  (void)host_records;
  (void)max_records;
  return PA_ERR_UNSUPPORTED;
#endif
}

extern "C" PA_API int pa_trace_clear(void) {
#if PA_TRACE
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, pa::g_trace) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemset(p, 0, sizeof(pa::TraceRecord) * pa::kTraceMax) != cudaSuccess) return PA_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
#else
  return PA_ERR_UNSUPPORTED;
#endif
}

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

extern "C" PA_API int pa_version(void) { return 102; }

extern "C" PA_API int pa_splitkv_num_partitions(int max_context_len, int partition_size) {
  if (partition_size <= 0) return 0;
  if (max_context_len <= 0) return 1;
  return static_cast<int>((static_cast<int64_t>(max_context_len) + partition_size - 1) / partition_size);
}

extern "C" PA_API size_t pa_splitkv_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                                    int max_context_len, int partition_size) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0 || partition_size <= 0)
    return 0;
  const int np = pa_splitkv_num_partitions(max_context_len, partition_size);
  pa::SplitkvLayout lay;
  if (!pa::splitkv_layout(static_cast<size_t>(num_seqs) * static_cast<size_t>(num_q_heads),
                          static_cast<size_t>(np), static_cast<size_t>(head_dim), &lay))
    return 0;
  return lay.total;
}
