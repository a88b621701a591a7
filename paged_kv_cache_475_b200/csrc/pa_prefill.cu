// Chunked prefill over a paged context: pa_prefill_chunk (tensor cores).
//
// Query i of a C-token chunk sits at position L - C + i and attends to keys
// 0..L-C+i: the whole earlier context and the chunk's own keys up to itself.
// This is eq. (4) of "Flash Attention vs Paged Attention" (算法原理: the block
// sum stops at the block holding the query, cut at its own token), evaluated
// with the online softmax and fused QK^T / softmax / PV of "FlashAttention y
// PagedAttention" (FlashAttention "Cómo funciona"); key tiles wholly past a
// query tile are never computed and the causal mask is applied in registers
// (kernel fusion section of the same Chinese page).
//
// Design: one CTA (4 warps) per (sequence, KV head, query tile). The 64 rows
// of a query tile are (query, head) pairs of one GQA group, so every K/V tile
// gathered from the pool serves all G heads. K/V tiles of 64 tokens are
// gathered page by page with 16-byte cp.async (zero-filled past the context),
// stored XOR-swizzled for conflict-free ldmatrix, double-buffered, and fed to
// bf16/f16 mma.sync m16n8k16 with fp32 accumulation.
#include "pa_common.cuh"

namespace pa {
namespace prefill {

constexpr int kBM = 64;   // query rows per CTA
constexpr int kBN = 64;   // keys per tile
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  unsigned int* err;
  int max_blocks, num_seqs, chunk, num_q_heads, num_kv_heads, block_size, num_blocks;
  float scale_log2;
};

__device__ inline void cp_async16(uint32_t dst, const void* src, bool fill) {
  const int n = fill ? 16 : 0;  // src-size 0: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ inline void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ inline void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ inline void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ inline void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <typename T> struct Mma;
template <> struct Mma<__nv_bfloat16> {
  __device__ static inline void run(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ static inline uint32_t pack(float x, float y) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  // Sum of the two rounded values in a packed pair (exact in fp32).
  __device__ static inline float sum2(uint32_t u) {
    return __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
  }
};
template <> struct Mma<__half> {
  __device__ static inline void run(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  __device__ static inline uint32_t pack(float x, float y) {
    __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static inline float sum2(uint32_t u) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    return f.x + f.y;
  }
};

// Byte offset of 16-byte chunk c of row r in a swizzled [rows][D] tile.
template <int D>
__device__ inline uint32_t swz(int r, int c) {
  constexpr int RC = D * 2 / 16;  // chunks per row
  return static_cast<uint32_t>(r * RC * 16 + ((c ^ (r & 7)) * 16));
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
prefill_kernel(const Params p) {
  constexpr int RC = D * 2 / 16;           // 16-byte chunks per row
  constexpr int QT = kBM / G;              // queries per CTA
  constexpr int KS = D / 16;               // k-steps over the head dim
  constexpr int NT = kBN / 8;              // score n-tiles per key tile
  constexpr int DT = D / 8;                // output n-tiles
  constexpr int kTileBytes = kBN * D * 2;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sQ = smem;
  unsigned char* sK = smem + kBM * D * 2;           // [2][kBN][D]
  unsigned char* sV = sK + 2 * kTileBytes;          // [2][kBN][D]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int num_qt = gridDim.x;
  const int qt = num_qt - 1 - blockIdx.x;   // heaviest (latest) query tiles first
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int C = p.chunk, B = p.block_size;

  int L = p.context_lens[b];
  if (L < 0 || L > p.max_blocks * B) {
    if (tid == 0) set_error(p.err, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : p.max_blocks * B;
  }
  const int i0 = qt * QT;                   // first query of the tile
  const int q_hi = min(C, i0 + QT);         // one past the last query
  const int pos_lo = L - C + i0;            // position of the first query
  const int pos_hi = L - C + q_hi - 1;      // position of the last query
  const int n_keys = pos_hi + 1 > 0 ? pos_hi + 1 : 0;
  const int n_ktiles = (n_keys + kBN - 1) / kBN;

  const T* qg = static_cast<const T*>(p.q);
  const T* kc = static_cast<const T*>(p.k_cache);
  const T* vc = static_cast<const T*>(p.v_cache);
  const int32_t* bt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;

  // ---- Q tile: row r = (query i0 + r/G, head kvh*G + r%G) -------------------
  for (int idx = tid; idx < kBM * RC; idx += kWarps * 32) {
    const int r = idx / RC, c = idx % RC;
    const int i = i0 + r / G;
    const bool ok = i < C;
    const T* src = qg + ((static_cast<int64_t>(b) * C + (ok ? i : 0)) * p.num_q_heads + kvh * G + r % G) * D + c * 8;
    cp_async16(smem_addr(sQ) + swz<D>(r, c), src, ok);
  }
  cp_async_commit();

  auto load_kv = [&](int kt, int buf) {
    const int t0 = kt * kBN;
    const uint32_t kbase = smem_addr(sK + buf * kTileBytes);
    const uint32_t vbase = smem_addr(sV + buf * kTileBytes);
    for (int idx = tid; idx < kBN * RC; idx += kWarps * 32) {
      const int r = idx / RC, c = idx % RC;
      const int t = t0 + r;
      bool ok = t < L;
      int64_t off = 0;
      if (ok) {
        const int id = bt[t / B];
        if (id < 0 || id >= p.num_blocks) {
          set_error(p.err, PA_DEVERR_BLOCK_ID);
          ok = false;
        } else {
          off = ((static_cast<int64_t>(id) * p.num_kv_heads + kvh) * B + t % B) * D + c * 8;
        }
      }
      cp_async16(kbase + swz<D>(r, c), kc + off, ok);
      cp_async16(vbase + swz<D>(r, c), vc + off, ok);
    }
  };

  if (n_ktiles > 0) load_kv(0, 0);
  cp_async_commit();

  // ---- per-thread row state ---------------------------------------------------
  const int r0 = warp * 16 + (lane >> 2);   // this thread's rows: r0 and r0 + 8
  const int pos_r0 = L - C + i0 + r0 / G;
  const int pos_r1 = L - C + i0 + (r0 + 8) / G;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[DT][4];
#pragma unroll
  for (int n = 0; n < DT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  uint32_t qa[KS][4];
  cp_async_wait<1>();
  __syncthreads();
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int r = warp * 16 + (lane & 15);
    const int c = ks * 2 + (lane >> 4);
    ldsm_x4(smem_addr(sQ) + swz<D>(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
  }

  for (int kt = 0; kt < n_ktiles; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < n_ktiles) load_kv(kt + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const uint32_t kb = smem_addr(sK + buf * kTileBytes);
    const uint32_t vb = smem_addr(sV + buf * kTileBytes);
    const int t0 = kt * kBN;

    // -- S = Q K^T (16 x 64 per warp) --
    float s[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = ks * 2 + ((lane >> 3) & 1);
        ldsm_x4(kb + swz<D>(r, c), b0, b1, b2, b3);
        Mma<T>::run(s[2 * np], qa[ks], b0, b1);
        Mma<T>::run(s[2 * np + 1], qa[ks], b2, b3);
      }
    }

    // -- causal mask (only tiles reaching past the first query's position) --
    const bool need_mask = t0 + kBN - 1 > pos_lo;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[n][e] * p.scale_log2;
        if (need_mask) {
          const int t = t0 + n * 8 + (lane & 3) * 2 + (e & 1);
          const int pr = e < 2 ? pos_r0 : pos_r1;
          if (t > pr) v = -INFINITY;
        }
        s[n][e] = v;
      }
    }

    // -- online softmax --
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
      mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = exp2f(m0 - mu0), a1 = exp2f(m1 - mu1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[NT / 2][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float p0 = exp2f(s[n][0] - mu0), p1 = exp2f(s[n][1] - mu0);
      const float p2 = exp2f(s[n][2] - mu1), p3 = exp2f(s[n][3] - mu1);
      // P enters the PV product rounded to the input type; the row sum is
      // taken over the same rounded values so the weights stay normalised.
      const uint32_t u01 = Mma<T>::pack(p0, p1), u23 = Mma<T>::pack(p2, p3);
      pa[n / 2][(n & 1) * 2 + 0] = u01;
      pa[n / 2][(n & 1) * 2 + 1] = u23;
      rs0 += Mma<T>::sum2(u01);
      rs1 += Mma<T>::sum2(u23);
    }
    l0 = l0 * a0 + rs0;
    l1 = l1 * a1 + rs1;
#pragma unroll
    for (int n = 0; n < DT; ++n) {
      o[n][0] *= a0; o[n][1] *= a0;
      o[n][2] *= a1; o[n][3] *= a1;
    }

    // -- O += P V --
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = dp * 2 + (lane >> 4);
        ldsm_x4_t(vb + swz<D>(r, c), b0, b1, b2, b3);
        Mma<T>::run(o[2 * dp], pa[kk], b0, b1);
        Mma<T>::run(o[2 * dp + 1], pa[kk], b2, b3);
      }
    }
    __syncthreads();  // buffer `buf` is refilled by the next iteration's load
  }
  cp_async_wait<0>();

  // ---- finish: O / l, written as (query, head) rows ---------------------------
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  T* out = static_cast<T*>(p.out);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = r0 + half * 8;
    const int i = i0 + r / G;
    if (i >= C) continue;
    const float inv = half ? inv1 : inv0;
    T* orow = out + ((static_cast<int64_t>(b) * C + i) * p.num_q_heads + kvh * G + r % G) * D;
#pragma unroll
    for (int n = 0; n < DT; ++n) {
      const int d = n * 8 + (lane & 3) * 2;
      const uint32_t v = Mma<T>::pack(o[n][half * 2] * inv, o[n][half * 2 + 1] * inv);
      *reinterpret_cast<uint32_t*>(orow + d) = v;
    }
  }
}

template <typename T, int D, int G>
int launch(const Params& prm, cudaStream_t s) {
  constexpr int QT = kBM / G;
  constexpr int kSmem = kBM * D * 2 + 4 * kBN * D * 2;
  auto kern = prefill_kernel<T, D, G>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
      return PA_ERR_CUDA;
    attr_done[dev] = true;
  }
  dim3 grid((prm.chunk + QT - 1) / QT, prm.num_kv_heads, prm.num_seqs);
  kern<<<grid, kWarps * 32, kSmem, s>>>(prm);
  return launch_status();
}

template <typename T, int D>
int by_group(const Params& prm, int G, cudaStream_t s) {
  switch (G) {
    case 1: return launch<T, D, 1>(prm, s);
    case 2: return launch<T, D, 2>(prm, s);
    case 4: return launch<T, D, 4>(prm, s);
    case 8: return launch<T, D, 8>(prm, s);
  }
  return PA_ERR_UNSUPPORTED;
}

template <typename T>
int by_dim(const Params& prm, int D, int G, cudaStream_t s) {
  if (D == 64) return by_group<T, 64>(prm, G, s);
  if (D == 128) return by_group<T, 128>(prm, G, s);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace prefill
}  // namespace pa

using namespace pa;

extern "C" PA_API int pa_prefill_chunk(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int max_blocks_per_seq,
                                       const int32_t* context_lens, int num_seqs, int chunk_len, int num_q_heads,
                                       int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                                       pa_dtype dtype, void* stream) {
  if (num_seqs < 0 || chunk_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks < 0 ||
      max_blocks_per_seq < 0)
    return PA_ERR_SHAPE;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_q_heads % num_kv_heads) return PA_ERR_SHAPE;
  const int G = num_q_heads / num_kv_heads;
  if (!supported_head_dim(head_dim) || !supported_block(block_size) || !supported_group(G))
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || chunk_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return PA_ERR_ALIGN;
  if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_SHAPE;
  prefill::Params prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.err = device_error_word();
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.chunk = chunk_len;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.scale_log2 = scale * prefill::kLog2e;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == PA_BF16) return prefill::by_dim<__nv_bfloat16>(prm, head_dim, G, s);
  return prefill::by_dim<__half>(prm, head_dim, G, s);
}
