// Merge of split-KV partials: pa_merge, and the merge step of the split-KV
// and shared-prefix paths in pa_decode.cu.
//
// What it computes: the combination of per-partition softmax states of
// eq. (4) of "Flash Attention vs Paged Attention" (算法原理): with m_p the
// partition's max score (natural-log units), l_p its sum of exp(s - m_p) and
// o_p its unnormalised output, out = sum_p exp(m_p - M) o_p / sum_p
// exp(m_p - M) l_p with M the largest live m_p. A partition is live when
// l_p > 0 (an empty one has m = -inf, l = 0) or when l_p is NaN, which is
// passed on as the definition does.
#include "pa_common.cuh"

#ifndef PA_MERGE_FEW
#define PA_MERGE_FEW 1  // rows with <= 8 live partitions: one warp per row (merge_few_kernel)
#endif

namespace pa {

// ---------------------------------------------------------------------------
// Merge of split-KV partials: one CTA of MW warps per (sequence, head).
// Pass 1 (all threads): M = max m_p and Lsum = sum exp(m_p - M) l_p over the
// live partitions. Pass 2: warp w accumulates exp(m_p - M) o_p for partitions
// w, w+MW, ...; the loads of successive partitions are independent, so many
// are in flight at once. The warps' sums meet in shared memory.
// ---------------------------------------------------------------------------
template <int MW>
__device__ inline float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmax_nan(v, o) : v + o;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < MW; ++w) r = is_max ? fmax_nan(r, red[w]) : r + red[w];
  __syncthreads();
  return r;
}

template <typename T, int D, int MW>
__global__ void __launch_bounds__(MW * 32)
merge_kernel(T* __restrict__ out, const float* __restrict__ part_o, const float* __restrict__ part_m,
             const float* __restrict__ part_l, const int32_t* __restrict__ context_lens, int num_q_heads,
             int partition, int num_parts) {
  constexpr int DPL = D / 32;
  __shared__ float s_o[MW][D];
  __shared__ float red[MW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x;  // b * Hq + h
  const int b = row / num_q_heads;
  // partition < 0 (cascade): the first -partition slots of each row are live
  int np = partition < 0 ? (-partition < num_parts ? -partition : num_parts) : num_parts;
  if (partition > 0) {
    int L = context_lens[b];
    L = L < 0 ? 0 : L;
    np = (L + partition - 1) / partition;
    np = np > num_parts ? num_parts : np;
  }
  const float* po = part_o + static_cast<int64_t>(row) * num_parts * D;
  const float* pm = part_m + static_cast<int64_t>(row) * num_parts;
  const float* pl = part_l + static_cast<int64_t>(row) * num_parts;

  float mloc = -INFINITY;
  for (int pp = threadIdx.x; pp < np; pp += MW * 32)
    if (!(pl[pp] <= 0.f)) mloc = fmax_nan(mloc, pm[pp]);  // live: l > 0, or NaN (passed on)
  const float M = block_reduce<MW>(mloc, red, true);
  float dloc = 0.f;
  if (M != -INFINITY)
    for (int pp = threadIdx.x; pp < np; pp += MW * 32) {
      const float l = pl[pp];
      dloc += !(l <= 0.f) ? expf(pm[pp] - M) * l : 0.f;
    }
  const float den = block_reduce<MW>(dloc, red, false);

  float o[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) o[j] = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int pp = warp; pp < np; pp += MW) {
      const float l = pl[pp];
      const float w = !(l <= 0.f) ? expf(pm[pp] - M) : 0.f;
      float v[DPL];
      if constexpr (DPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(po + static_cast<int64_t>(pp) * D + lane * 4);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(po + static_cast<int64_t>(pp) * D + lane * 2);
        v[0] = x.x; v[1] = x.y;
      }
#pragma unroll
      for (int j = 0; j < DPL; ++j) o[j] += !(l <= 0.f) ? w * v[j] : 0.f;
    }
  }
#pragma unroll
  for (int j = 0; j < DPL; ++j) s_o[warp][lane * DPL + j] = o[j];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += MW * 32) {
    float num = 0.f;
#pragma unroll
    for (int w = 0; w < MW; ++w) num += s_o[w][d];
    out[static_cast<int64_t>(row) * D + d] = Elem<T>::from_f(!(den <= 0.f) ? num / den : 0.f);
  }
}

// Merge of rows with at most PMAX live partitions (the shared-prefix cascade:
// prefix splits + suffix; short split-KV rows): one warp per (sequence, head)
// row, 8 rows per CTA. Every load of a row (its context length, m and l of
// each partition, this lane's D/32 output dims of each partition) is issued
// before any is used, so a row costs one round trip to memory; partitions
// past the row's live count are loaded (in bounds: the row holds num_parts)
// and then ignored. Same arithmetic as merge_kernel: M over the live
// partitions (l > 0, or NaN, which is passed on), weights exp(m_p - M),
// out = sum w_p o_p / sum w_p l_p.
template <typename T, int D, int PMAX>
__global__ void __launch_bounds__(256)
merge_few_kernel(T* __restrict__ out, const float* __restrict__ part_o, const float* __restrict__ part_m,
                 const float* __restrict__ part_l, const int32_t* __restrict__ context_lens, int rows,
                 int num_q_heads, int partition, int num_parts) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const int b = row / num_q_heads;
  const int nload = num_parts < PMAX ? num_parts : PMAX;
  const float* po = part_o + static_cast<int64_t>(row) * num_parts * D + lane * DPL;
  const float* pm = part_m + static_cast<int64_t>(row) * num_parts;
  const float* pl = part_l + static_cast<int64_t>(row) * num_parts;

  const int L = partition > 0 ? context_lens[b] : 0;
  float m = -INFINITY, l = 0.f;
  if (lane < nload) {
    m = pm[lane];
    l = pl[lane];
  }
  float v[PMAX][DPL];
#pragma unroll
  for (int pp = 0; pp < PMAX; ++pp) {
    if (pp < nload) {
      if constexpr (DPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(po + static_cast<int64_t>(pp) * D);
        v[pp][0] = x.x; v[pp][1] = x.y; v[pp][2] = x.z; v[pp][3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(po + static_cast<int64_t>(pp) * D);
        v[pp][0] = x.x; v[pp][1] = x.y;
      }
    } else {
#pragma unroll
      for (int j = 0; j < DPL; ++j) v[pp][j] = 0.f;
    }
  }
  // partition < 0 (cascade): the first -partition slots are live
  int np = partition < 0 ? (-partition < nload ? -partition : nload) : nload;
  if (partition > 0) {
    const int Lc = L < 0 ? 0 : L;
    const int need = (Lc + partition - 1) / partition;
    np = need < np ? need : np;
  }
  const bool live = lane < np && !(l <= 0.f);
  float M = live ? m : -INFINITY;
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) M = fmax_nan(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float w = (live && M != -INFINITY) ? expf(m - M) : 0.f;
  float den = live ? w * l : 0.f;  // l of a slot past the live ones may be anything, NaN included
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(0xffffffffu, den, off);
  float o[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) o[j] = 0.f;
#pragma unroll
  for (int pp = 0; pp < PMAX; ++pp) {
    const float wp = __shfl_sync(0xffffffffu, w, pp);
    const bool lp = __shfl_sync(0xffffffffu, live ? 1 : 0, pp) != 0;
#pragma unroll
    for (int j = 0; j < DPL; ++j) o[j] += lp ? wp * v[pp][j] : 0.f;
  }
  T* dst = out + static_cast<int64_t>(row) * D + lane * DPL;
#pragma unroll
  for (int j = 0; j < DPL; ++j) dst[j] = Elem<T>::from_f(!(den <= 0.f) ? o[j] / den : 0.f);
}

template <typename T, int MW>
int launch_merge_mw(void* out, const float* po, const float* pm, const float* pl, const int32_t* lens, int rows,
                    int Hq, int D, int partition, int np, cudaStream_t s) {
  if (D == 64)
    merge_kernel<T, 64, MW><<<rows, MW * 32, 0, s>>>(static_cast<T*>(out), po, pm, pl, lens, Hq, partition, np);
  else if (D == 128)
    merge_kernel<T, 128, MW><<<rows, MW * 32, 0, s>>>(static_cast<T*>(out), po, pm, pl, lens, Hq, partition, np);
  else
    return PA_ERR_UNSUPPORTED;
  return launch_status();
}
// 8 warps per row when there are many partitions, 2 when there are few.
template <typename T>
int launch_merge(void* out, const float* po, const float* pm, const float* pl, const int32_t* lens, int rows,
                 int Hq, int D, int partition, int np, cudaStream_t s) {
  const int live = partition < 0 ? -partition : np;
#if PA_MERGE_FEW
  if (live <= 8) {
    const int grid = (rows + 7) / 8;
    if (D == 64)
      merge_few_kernel<T, 64, 8><<<grid, 256, 0, s>>>(static_cast<T*>(out), po, pm, pl, lens, rows, Hq, partition, np);
    else if (D == 128)
      merge_few_kernel<T, 128, 8><<<grid, 256, 0, s>>>(static_cast<T*>(out), po, pm, pl, lens, rows, Hq, partition, np);
    else
      return PA_ERR_UNSUPPORTED;
    return launch_status();
  }
#endif
  if (live <= 8) return launch_merge_mw<T, 2>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
  if (live <= 64) return launch_merge_mw<T, 8>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
  return launch_merge_mw<T, 32>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
}
}  // namespace pa

using namespace pa;

extern "C" PA_API int pa_merge(void* out, const float* part_o, const float* part_m, const float* part_l,
                               const int32_t* context_lens, int num_seqs, int num_q_heads, int head_dim,
                               int partition_size, int num_partitions, pa_dtype dtype, void* stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_partitions <= 0) return PA_ERR_SHAPE;
  if (!supported_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
  if (partition_size <= 0) return PA_ERR_WORKSPACE;
  if (num_seqs == 0) return PA_OK;
  if (!out || !part_o || !part_m || !part_l || !context_lens) return PA_ERR_NULL;
  if (!aligned16(part_o)) return PA_ERR_ALIGN;
  const int64_t rows = static_cast<int64_t>(num_seqs) * num_q_heads;
  if (rows > 0x7fffffff) return PA_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  switch (dtype) {
    case PA_F32: return launch_merge<float>(out, part_o, part_m, part_l, context_lens, (int)rows, num_q_heads,
                                            head_dim, partition_size, num_partitions, s);
    case PA_F16: return launch_merge<__half>(out, part_o, part_m, part_l, context_lens, (int)rows, num_q_heads,
                                             head_dim, partition_size, num_partitions, s);
    case PA_BF16: return launch_merge<__nv_bfloat16>(out, part_o, part_m, part_l, context_lens, (int)rows,
                                                     num_q_heads, head_dim, partition_size, num_partitions, s);
  }
  return PA_ERR_DTYPE;
}

namespace pa {
int launch_merge_any(void* out, const float* po, const float* pm, const float* pl, const int32_t* lens, int rows,
                     int Hq, int D, int partition, int np, pa_dtype dt, cudaStream_t s) {
  switch (dt) {
    case PA_F32: return launch_merge<float>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
    case PA_F16: return launch_merge<__half>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
    case PA_BF16: return launch_merge<__nv_bfloat16>(out, po, pm, pl, lens, rows, Hq, D, partition, np, s);
  }
  return PA_ERR_DTYPE;
}
}  // namespace pa
