// Shared device helpers for the paged-KV attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// ---------------------------------------------------------------------------
// Host-side helpers
// ---------------------------------------------------------------------------

// Device error word of the current device (lives in pa_api.cu).
unsigned int* device_error_word();

// Identity of the CUDA context current on this host thread, unique over the
// life of the process; 0 when no context is current or the driver cannot say.
// A device reset destroys the primary context and with it every address of a
// module-scope __device__ variable and every function attribute set in it, so
// per-device caches of those remember the context they were taken in.
uint64_t current_context_id();

// A per-device cached value, valid only in the context it was taken in.
template <typename V>
struct ContextCached {
  uint64_t ctx = 0;
  V value{};
  bool valid() const {
    const uint64_t now = current_context_id();
    return now != 0 && now == ctx;
  }
  void set(V v) {
    value = v;
    ctx = current_context_id();
  }
};

// Byte layout of a split-KV workspace holding part_o [rows, np, D] at offset
// 0, part_m [rows, np] at o_bytes and part_l [rows, np] at o_bytes + ml_bytes
// (rows = N * Hq), each part rounded up to a multiple of 256 bytes. Returns
// false when a size does not fit in size_t.
struct SplitkvLayout {
  size_t o_bytes = 0, ml_bytes = 0, total = 0;
};
inline bool splitkv_layout(size_t rows, size_t np, size_t head_dim, SplitkvLayout* out) {
  constexpr size_t kMax = ~size_t(0);
  if (rows != 0 && np > kMax / rows) return false;
  const size_t cells = rows * np;
  const size_t row_bytes = head_dim * sizeof(float);
  if (row_bytes != 0 && cells > (kMax - 255) / row_bytes) return false;
  if (cells > (kMax - 255) / sizeof(float)) return false;
  const size_t o = (cells * row_bytes + 255) & ~size_t(255);
  const size_t ml = (cells * sizeof(float) + 255) & ~size_t(255);
  if (ml > (kMax - o) / 2) return false;
  out->o_bytes = o;
  out->ml_bytes = ml;
  out->total = o + 2 * ml;
  return true;
}

// Shared-prefix mode of the tensor-core prefill kernel: the group's decode
// queries attend to keys [0, prefix_len) of block-table row 0, cut into
// key_splits ranges, and the results land as split-KV partials in slots
// 0..key_splits-1 of [N, Hq, num_partitions, D].
struct PrefixPartials {
  int prefix_len;
  float* part_o;
  float* part_m;
  float* part_l;
  int num_partitions;
  int key_splits;  // the prefix keys are cut into this many equal ranges, one partial slot each
};

int prefill_tcgen05(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int chunk_len,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                    pa_dtype dtype, cudaStream_t stream, const PrefixPartials* pp);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool supported_block(int b) { return b == 8 || b == 16 || b == 32 || b == 64 || b == 128; }
inline bool supported_head_dim(int d) { return d == 64 || d == 128; }
inline bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

inline int dtype_bytes(pa_dtype dt) { return dt == PA_F32 ? 4 : 2; }

// Records the message of the last failing CUDA call of this host thread
// (read back with pa_last_cuda_error) and maps it to PA_ERR_CUDA.
int record_cuda_error(cudaError_t e, const char* where);

inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : record_cuda_error(e, "kernel launch");
}

// ---------------------------------------------------------------------------
// Element types
// ---------------------------------------------------------------------------

template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kBytes = 4;
  __device__ static inline float to_f(float x) { return x; }
  __device__ static inline float from_f(float x) { return x; }
};
template <> struct Elem<__half> {
  static constexpr int kBytes = 2;
  __device__ static inline float to_f(__half x) { return __half2float(x); }
  __device__ static inline __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  __device__ static inline float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static inline __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Unpack a 16-byte chunk into floats (8 halves / 8 bf16 / 4 floats).
__device__ inline void unpack16(const uint4& u, float* f, float) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}
__device__ inline void unpack16(const uint4& u, float* f, __half) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 v = __half22float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}
__device__ inline void unpack16(const uint4& u, float* f, __nv_bfloat16) {
  // bf16 -> fp32 is exact: the bf16 bits are the high half of the float.
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Unpack 2 x 32-bit words (8 bytes).
__device__ inline void unpack8(const uint2& u, float* f, float) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
}
__device__ inline void unpack8(const uint2& u, float* f, __half) {
  float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}
__device__ inline void unpack8(const uint2& u, float* f, __nv_bfloat16) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
}
// Unpack one 32-bit word (2 halves / 2 bf16 / 1 float).
__device__ inline void unpack4(uint32_t u, float* f, float) { f[0] = __uint_as_float(u); }
__device__ inline void unpack4(uint32_t u, float* f, __half) {
  float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u));
  f[0] = a.x; f[1] = a.y;
}
__device__ inline void unpack4(uint32_t u, float* f, __nv_bfloat16) {
  f[0] = __uint_as_float(u << 16);
  f[1] = __uint_as_float(u & 0xffff0000u);
}

// ---------------------------------------------------------------------------
// Shared-memory barriers and bulk (TMA 1-D) copies, inline PTX
// ---------------------------------------------------------------------------

__device__ inline uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ inline void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// Bounded wait on a phase of an mbarrier: gives up after about `max_cycles`
// SM clock cycles (~2 s at 1.9 GHz by default), however long each try_wait
// suspends. Returns false on timeout (the caller records PA_DEVERR_WAIT).
__device__ inline bool mbar_try(uint32_t a, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(a), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, long long max_cycles = 4000000000LL) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try(a, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(a, parity)) return true;
    if (clock64() - t0 > max_cycles) return false;
  }
}

// Global -> shared bulk copy completing on an mbarrier (byte count, 16-byte
// aligned addresses and size). L2 hint: evict-first (KV pages are streamed once).
__device__ inline void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_addr(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ inline uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ inline void set_error(unsigned int* err, unsigned int bit) {
  if (err) atomicOr(err, bit);
}

// ---------------------------------------------------------------------------
// Timeline tracing (builds with -DPA_TRACE=1 only; off by default). A traced
// kernel stamps, per CTA, the global timer at entry, when its first tile has
// landed, and at exit, with the SM it ran on and the work it did; the records
// go to a fixed device array that pa_trace_read copies out.
// ---------------------------------------------------------------------------
#ifndef PA_TRACE
#define PA_TRACE 0
#endif
struct TraceRecord {
  unsigned long long t_start, t_first, t_end;  // %globaltimer, ns
  int smid, seq, kv_head, part, tokens, kind;
};
constexpr int kTraceMax = 1 << 16;
// Device address of the record array (lives in pa_api.cu; every .cu is its own
// device module, so kernels get the address as a parameter); null unless PA_TRACE.
TraceRecord* trace_buffer();

// Merge of split-KV partials (pa_merge.cu) on `s`, for `rows` = N * Hq rows;
// partition < 0: the first -partition slots of each row are live.
int launch_merge_any(void* out, const float* po, const float* pm, const float* pl, const int32_t* lens, int rows,
                     int Hq, int D, int partition, int np, pa_dtype dt, cudaStream_t s);
#if PA_TRACE
__device__ inline unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ inline int sm_id() {
  int s;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
  return s;
}
#endif

// Packed fp32 FMA (sm_100): {a.x*b.x + c.x, a.y*b.y + c.y} in one instruction.
__device__ inline float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Maximum that returns NaN when either input is NaN (fmaxf returns the other
// one), so that a NaN score or partial reaches the output as in the
// definition of softmax attention instead of dropping out of a running max.
__device__ inline float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

}  // namespace pa
