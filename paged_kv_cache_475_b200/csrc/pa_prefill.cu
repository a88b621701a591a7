// Chunked prefill over a paged context on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), sm_100a.
//
// What it computes (pa_prefill_chunk in include/pa.h): query
// i of a C-token chunk sits at position L - C + i and attends to keys
// 0..L-C+i; eq. (4) of "Flash Attention vs Paged Attention" (算法原理) with the
// online softmax and fused QK^T / softmax / PV of "FlashAttention y
// PagedAttention" (FlashAttention "Cómo funciona"); key tiles past a query
// tile are never computed, the causal mask is applied in registers.
//
// One CTA (7 warps) per (sequence, KV head, 128-row query tile), two CTAs per
// SM; the 128 rows are (query, head) pairs of one GQA group, so each gathered
// K/V page serves all G heads of the group. Warp roles:
//   warps 0-3  softmax: warp w owns rows 32w.. (its TMEM lanes) and all 64 keys
//              of every tile: one online-softmax stream per row (running max
//              and sum in registers, O in TMEM), P (bf16/f16) written back into
//              TMEM over the S columns it read, O rescaled only when the row
//              max grows by more than 2^8;
//   warps 4,6  producers: TMA tensor copies of the Q tile (once) and of each
//              64-key K tile (warp 4) and V tile (warp 6, its own ring), one
//              box per lane, addressed through the CTA's block-table entries
//              (each read one tile ahead of its copy; PA_TC_BT_STAGED > 0
//              stages the first ones in shared memory instead, measured
//              slower) with one 2-D box of min(B,16) rows per page chunk and
//              128-byte atom, 128-byte swizzle; chunks past the context read
//              out of range as zeros;
//   warp 5     MMA: one thread issues S = Q K^T (M = 128, N = 64) into a
//              double-buffered TMEM accumulator and O += P V (P read straight
//              from TMEM as the A operand, K = 16 per instruction), completions
//              by tcgen05.commit on mbarriers; it zeroes V rows past the context
//              in the last partial page chunk before they reach the PV product.
// A single CTA's tile chain is serial (S(j+2) needs PV(j), which needs the
// softmax's P(j)), so each CTA holds half of what one CTA per SM would (256 TMEM
// columns, 96 KB of shared memory) and the SM interleaves two such chains on
// its tensor pipe. Per 64-key tile the MMA thread issues 12 instructions of
// 24-47 ns of tensor work each, and issuing them takes about 0.7 us of the
// ~1.25 us tile period: with tiles this size the issuing thread, not the
// tensor pipe, sets the pace.
// Every mbarrier wait is bounded; a timeout sets PA_DEVERR_WAIT and the CTA
// drains, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "pa_common.cuh"

namespace pa {
namespace tc {

constexpr int kM = 128;        // query rows per CTA = TMEM lanes
constexpr int kN = 64;         // keys per tile
#ifndef PA_TC_KSTAGES
#define PA_TC_KSTAGES 2
#endif
#ifndef PA_TC_VSTAGES
#define PA_TC_VSTAGES 2
#endif
#ifndef PA_TC_SMEM_SLACK
#define PA_TC_SMEM_SLACK 0  // bytes reserved to align the dynamic shared-memory base at run time (the base
                            // measured 1024-aligned; the kernel checks it and reports PA_DEVERR_SETUP if not)
#endif
constexpr int kStagesK = PA_TC_KSTAGES;  // K ring (16 KB per stage at D = 128)
constexpr int kStagesV = PA_TC_VSTAGES;  // V ring
#ifndef PA_TC_SLOT_BY_COMPLETION
// With two-slot rings a K slot is free once the S two tiles back has
// completed, and a V slot once the PV two tiles back has: the producers wait
// on those barriers (s_full / o_done), so the MMA thread issues no commit of
// its own to release a slot.
#define PA_TC_SLOT_BY_COMPLETION 1
#endif
static_assert(!PA_TC_SLOT_BY_COMPLETION || (kStagesK == 2 && kStagesV == 2),
              "slot release through s_full / o_done needs two-slot rings");
#ifndef PA_TC_BT_STAGED
#define PA_TC_BT_STAGED 0  // block-table entries staged in shared memory (0: each read one tile ahead; 128 / 256 / 1024 measured 1 / 2 / 3% slower)
#endif
constexpr int kBtStaged = PA_TC_BT_STAGED;
constexpr int kThreads = 224;  // 4 softmax warps + K producer + MMA + V producer
constexpr int kProducerWarp = 4;   // Q once, then K tiles
constexpr int kMmaWarp = 5;
constexpr int kVProducerWarp = 6;  // V tiles
constexpr int kTmemCols = 256;     // S double buffer [0, 128), O [128, 128 + D); two CTAs share an SM's 512
constexpr int kCtasPerSm = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // keep a stale max until the true one is 2^8 larger

struct Params {
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  unsigned int* err;
  int max_blocks, num_seqs, chunk, num_q_heads, num_kv_heads, block_size, num_blocks;
  int chunk_rows;      // rows per TMA box = min(B, 16)
  int oob_row;         // a row coordinate past the pool: TMA reads zeros there
  float scale_log2;
  // Shared-prefix mode (prefix_len > 0): the "chunk" is a group of decode
  // queries (one per sequence) that all see keys [0, prefix_len) of block
  // table row 0, without a causal mask; the result is written as split-KV
  // partials (slot 0 of [N, Hq, part_np, D]) instead of normalised rows.
  int prefix_len;
  float* part_o;
  float* part_m;
  float* part_l;
  int part_np;
  int key_splits;
  TraceRecord* trace;  // per-role timeline of one CTA (PA_TRACE builds), else null
};

// Per-role timeline events of the traced CTA (PA_TRACE builds): record index
// event * 256 + tile, t_start = the global timer, kind = 100 + event.
enum TraceEvent {
  kEvKSlotFree = 0,  // K producer: slot free (empty barrier passed)
  kEvKIssued,        // K producer: the tile's copies issued
  kEvVSlotFree,      // V producer
  kEvVIssued,
  kEvMmaKFull,       // MMA: K tile landed
  kEvMmaSIssued,     // MMA: S = Q K^T issued
  kEvMmaVFull,       // MMA: V tile landed
  kEvMmaP0,          // MMA: P ready
  kEvMmaP1,          // (unused)
  kEvMmaPVIssued,    // MMA: both halves of P V issued
  kEvSm0SFull,       // softmax warp 0 (rows 0..31): S ready
  kEvSm0PStored,     // softmax warp 0: P stored and signalled
  kEvSm4SFull,       // softmax warp 1 (rows 32..63)
  kEvSm4PStored,
  kEvKRowsDone,      // K producer: row coordinates of the tile computed
  kEvKExpectDone,    // K producer: expect_tx armed, warp synchronised
  kEvKAtom0Issued,   // K producer: copies of the first 64 columns issued
};

template <int D>
struct Smem {
  static constexpr int kQ = kM * D * 2;   // D/64 atoms of [128 rows x 128 B]
  static constexpr int kKV = kN * D * 2;  // one K or V tile: D/64 atoms of [64 rows x 128 B]
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQ;
  static constexpr int oV = oK + kStagesK * kKV;
  static constexpr int oBar = oV + kStagesV * kKV;
  // q_full, k_full/k_empty[SK], v_full/v_empty[SV], s_full[2], p_full[2], o_done[2], bt_ready
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 2 + 2 + 2 + 1;
  static constexpr int oTmem = oBar + kNumBars * 8;
  // The CTA's block-table entries as TMA row coordinates, staged once.
  static constexpr int oBt = (oTmem + 16 + 15) & ~15;
  static constexpr int kUsed = oBt + 4 * (kBtStaged > 0 ? kBtStaged : 1);
  static constexpr int kAlloc = kUsed + PA_TC_SMEM_SLACK;  // room to align the base to 1024 B
};

// ---------------------------------------------------------------------------
// tcgen05 / TMA wrappers (inline PTX)
// ---------------------------------------------------------------------------
__device__ inline void tmem_alloc(uint32_t* slot, int cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(cols)
               : "memory");
}
__device__ inline void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ inline void tmem_dealloc(uint32_t taddr, int cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ inline void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ inline void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// Barrier over `count` threads (whole warps) with id `id`; returns the AND of
// `pred` over them, so every participant takes the same branch afterwards.
__device__ inline bool pair_and(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16, one CTA.
__device__ inline void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16, one CTA: A (M x K, K-major)
// lives in TMEM, row i in lane i, two 16-bit elements per 32-bit column.
__device__ inline void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ inline void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ inline void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ inline void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ inline void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ inline void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
__device__ inline void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
// lbo/sbo in 16-byte units.
__device__ inline uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(lbo & 0x3FFFu) << 16) |
         (static_cast<uint64_t>(sbo & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, A/B both `fmt`
// (0 = f16, 1 = bf16), A K-major, B K-major (b_mn = 0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t fmt, uint32_t b_mn, int M, int N) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | (b_mn << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// 2^x for the softmax. The MUFU unit computes one ex2 per lane-cycle on a
// pipe 8x narrower than the FMA pipe, and the softmax needs one per score, so
// a share of the exponentials is computed on the FMA pipe instead (the
// FMA-offload idea published with FlashAttention-4):
//   x = j + f, j = round(x) by the 1.5 * 2^23 rounding trick, f in [-1/2, 1/2];
//   2^f ~ c0 + c1 f + c2 f^2 + c3 f^3, coefficients fitted by this library
//   (weighted least squares on Chebyshev nodes, max relative error 7.5e-5 on
//   [-1/2, 1/2], far below the rounding of P to bf16/f16);
//   2^j is added to the exponent field of the result (as in Schraudolph's
//   exponent-field construction). x is clamped to [-125, 125] so the result
//   stays a normal float, and anything below -125 (masked scores, -inf)
//   returns exactly 0 like ex2.approx.ftz does.
// ---------------------------------------------------------------------------
#ifndef PA_TC_POLY_OF_4
#define PA_TC_POLY_OF_4 0  // pairs of scores out of every 4 that take the FMA path (0 measured fastest)
#endif
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716648042202f;

__device__ inline float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float ex2_fma(float x) {
  const bool zero = !(x >= -125.f);
  x = fminf(fmaxf(x, -125.f), 125.f);
  const float y = x + 12582912.f;  // 1.5 * 2^23: the low mantissa bits of y hold round(x)
  const float j = y - 12582912.f;
  const float f = x - j;
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return zero ? 0.f : __int_as_float(__float_as_int(p) + (__float_as_int(y) << 23));
}
template <bool kFma>
__device__ inline float ex2_sel(float x) {
  if constexpr (kFma) return ex2_fma(x);
  else return ex2_mufu(x);
}

template <typename T> struct Fmt;
#ifndef PA_TC_INT_PACK
#define PA_TC_INT_PACK 0  // the cvt pack measured faster (624 vs 601 TFLOP/s)
#endif
template <> struct Fmt<__nv_bfloat16> {
  static constexpr uint32_t kCode = 1;
  __device__ static inline uint32_t pack(float x, float y) {
#if PA_TC_INT_PACK
    // Round-to-nearest-even to bf16 with integer ops (ALU pipe, keeping the
    // conversion off the MUFU/XU pipe that the exponentials saturate). Valid
    // for the finite, non-negative probabilities this is used on.
    uint32_t ux = __float_as_uint(x), uy = __float_as_uint(y);
    ux += 0x7fffu + ((ux >> 16) & 1u);
    uy += 0x7fffu + ((uy >> 16) & 1u);
    return __byte_perm(ux, uy, 0x7632);
#else
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&h);
#endif
  }
  // Round-to-nearest-even of any fp32 pair (used for the output rows).
  __device__ static inline uint32_t pack_any(float x, float y) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static inline float sum2(uint32_t u) {
    return __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
  }
  __device__ static inline float2 unpack2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
};
template <> struct Fmt<__half> {
  static constexpr uint32_t kCode = 0;
  __device__ static inline uint32_t pack(float x, float y) {
    __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static inline uint32_t pack_any(float x, float y) { return pack(x, y); }
  __device__ static inline float sum2(uint32_t u) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    return f.x + f.y;
  }
  __device__ static inline float2 unpack2(uint32_t u) { return __half22float2(*reinterpret_cast<const __half2*>(&u)); }
};

// Every wait of this kernel gives up after about 2 s and is made warp-uniform,
// so a timeout can never split a warp at a __syncwarp.
__device__ inline bool wait_all(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

template <typename T, int D, int G>
// 7 warps per CTA, two CTAs per SM: 448 threads, so up to 146 registers each.
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using S = Smem<D>;
  constexpr int QT = kM / G;       // queries per CTA
  constexpr int KA = D / 64;       // 128-byte atoms along the head dim
  constexpr int KS = D / 16;       // MMA k-steps of S = Q K^T
  constexpr int KP = kN / 16;      // MMA k-steps of O += P V
  constexpr uint32_t kIdescS = idesc_f16(Fmt<T>::kCode, 0, kM, kN);
  constexpr uint32_t kIdescO = idesc_f16(Fmt<T>::kCode, 1, kM, D);

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  // The 128-byte-swizzled tiles need a 1024-byte-aligned base. Without the
  // slack to align it here, a base that is not aligned is reported and the
  // CTA does nothing (checked before any shared memory or TMEM is touched).
  if (PA_TC_SMEM_SLACK < 1024 && (raw_addr & 1023u) != 0u) {
    if (threadIdx.x == 0) set_error(p.err, PA_DEVERR_SETUP);
    return;
  }
  unsigned char* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sb = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::oBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStagesK;
  uint64_t* v_full = k_empty + kStagesK;
  uint64_t* v_empty = v_full + kStagesV;
  uint64_t* s_full = v_empty + kStagesV;  // [2]: S of tile 2n+u in buffer u (phase n)
  // p_full[u]: P of tile 2n+u written over buffer u (phase n); one barrier per
  // buffer, so the softmax can never be two phases ahead of the MMA's wait.
  uint64_t* p_full = s_full + 2;
  // o_done[u]: PV of tile 2n+u done (phase n). One barrier per buffer, like
  // p_full: a waiter knows only that PV(j-2) is done when it waits for
  // PV(j) (S(j) was issued after it), so with a single barrier it could be two
  // phases behind and a parity wait would return on the older phase.
  uint64_t* o_done = p_full + 2;
  uint64_t* bt_ready = o_done + 2;  // the staged block-table entries are in (32 arrivals)
  int32_t* bt_s = reinterpret_cast<int32_t*>(smem + S::oBt);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::oTmem);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // latest (heaviest) query tiles first
#if PA_TRACE
  // the traced CTA: the first dispatched (heaviest query tile) of sequence 0, KV head 0
  const bool tr_on = p.trace != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
#define PA_TR(ev, j)                                                                                   \
  do {                                                                                                 \
    if (tr_on && lane == 0 && (j) < 256)                                                               \
      p.trace[(ev) * 256 + (j)] = TraceRecord{global_ns(), 0, 0, sm_id(), (j), 0, 0, 0, 100 + (ev)};   \
  } while (0)
#else
#define PA_TR(ev, j) do { } while (0)
#endif
  const bool prefix_mode = p.prefix_len > 0;
  // prefix mode: z selects one of key_splits equal key ranges [key0, key0 + per)
  const int kvh = blockIdx.y, b = prefix_mode ? 0 : static_cast<int>(blockIdx.z);
  const int split = prefix_mode ? static_cast<int>(blockIdx.z) : 0;
  const int C = p.chunk, B = p.block_size;
  const int per = prefix_mode ? p.prefix_len / p.key_splits : 0;
  const int key0 = split * per;                 // first key of this CTA's range (0 when causal)
  int L = prefix_mode ? key0 + per : p.context_lens[b];  // keys [key0, L)
  if (L < 0 || L > p.max_blocks * B) {
    if (threadIdx.x == 0) set_error(p.err, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : p.max_blocks * B;
  }
  const int i0 = qt * QT;
  const int q_hi = min(C, i0 + QT);
  // causal: query i at position L - C + i; prefix mode: every query sees all keys of the range
  const int pos_lo = prefix_mode ? L - 1 : L - C + i0;
  const int pos_hi = prefix_mode ? L - 1 : L - C + q_hi - 1;
  const int n_keys = pos_hi + 1 > key0 ? pos_hi + 1 - key0 : 0;
  const int n_tiles = (n_keys + kN - 1) / kN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
    mbar_init(bt_ready, 32);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S (double buffer) [0, 2 kN), O [2 kN, 2 kN + D).
  const uint32_t tS0 = tmem, tS1 = tmem + kN;
  const uint32_t tO = tmem + 2 * kN;

  const uint32_t sQ = sb + S::oQ, sK = sb + S::oK, sV = sb + S::oV;
  const int32_t* bt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;

  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ------------------------- producers (K and V) -------------------------
    // One warp per ring, one TMA box per lane: a tile is kN / R page chunks
    // of R = min(B, 16) rows times D / 64 swizzle atoms, all issued by one
    // warp instruction.
    const bool is_k = warp == kProducerWarp;
    if (n_tiles > 0) {
      if (is_k && lane == 0) {
        mbar_arrive_expect_tx(q_full, S::kQ);
        for (int a = 0; a < KA; ++a)
          tma_load_3d(sQ + a * (kM * 128), &tm_q, a * 64, kvh * G, b * C + i0, q_full);
      }
      const int R = p.chunk_rows;
      const int chunks = kN / R;
      const int stages = is_k ? kStagesK : kStagesV;
      int n_tiles_local = n_tiles;
      uint64_t* full = is_k ? k_full : v_full;
#if !PA_TC_SLOT_BY_COMPLETION
      uint64_t* empty = is_k ? k_empty : v_empty;
#endif
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      const uint32_t ring = is_k ? sK : sV;
      // The CTA's pages [jb0, jb0 + n_bt) as TMA row coordinates, staged
      // once in shared memory (the first kBtStaged of them): row (id * Hkv +
      // kvh) * B of the pool viewed as [P * Hkv * B, D], or -1 for a bad id.
      // The K producer's lanes fill it and each arrives on bt_ready after its
      // own stores; the V producer waits for that. Per-tile lookups then read
      // shared memory instead of waiting on global loads that queue behind
      // the tiles' own traffic.
      const int jb0 = key0 / B;
      const int k_end = min(L, key0 + n_tiles * kN);
      const int n_bt = k_end > key0 ? (k_end - 1) / B - jb0 + 1 : 0;
      const int n_staged = n_bt < kBtStaged ? n_bt : kBtStaged;
      auto page_row = [&](int id) -> int {
        if (id >= 0 && id < p.num_blocks) return (id * p.num_kv_heads + kvh) * B;
        set_error(p.err, PA_DEVERR_BLOCK_ID);
        return -1;
      };
      if (is_k) {
        for (int i = lane; i < n_staged; i += 32) bt_s[i] = page_row(bt[jb0 + i]);
        mbar_arrive(bt_ready);
      } else if (!wait_all(bt_ready, 0)) {
        if (lane == 0) set_error(p.err, PA_DEVERR_WAIT);
        n_tiles_local = 0;
      }
      __syncwarp();
      // This lane's box of every tile: page chunk c, atom a.
      const bool has_box = lane < chunks * KA;
      const int c = has_box ? lane % chunks : 0;
      const int a = has_box ? lane / chunks : 0;
      auto row_of = [&](int j) -> int {
        int y = p.oob_row;  // chunks past the context read out of range: zeros
        const int t0 = key0 + j * kN + c * R;
        if (has_box && j < n_tiles && t0 < L) {
          const int jj = t0 / B - jb0;
          const int row = jj < n_staged ? bt_s[jj] : page_row(bt[t0 / B]);
          if (row >= 0) y = row + (t0 % B);
        }
        return y;
      };
      int y_next = row_of(0);
      for (int j = 0; j < n_tiles_local; ++j) {
        const int st = j % stages;
        const int y = y_next;
        y_next = row_of(j + 1);  // issued before the wait, so a global lookup's latency hides behind it
#if PA_TC_SLOT_BY_COMPLETION
        // slot st last held tile j - 2: free once S(j - 2) (K) or PV(j - 2) (V)
        // has completed, phase (j - 2) / 2 of that tile's buffer barrier
        if (j >= 2 && !wait_all(is_k ? &s_full[j & 1] : &o_done[j & 1], ((j - 2) >> 1) & 1)) {
#else
        if (!wait_all(&empty[st], ((j / stages) & 1) ^ 1)) {
#endif
          if (lane == 0) set_error(p.err, PA_DEVERR_WAIT);
          break;
        }
        PA_TR(is_k ? kEvKSlotFree : kEvVSlotFree, j);
        if (lane == 0) mbar_arrive_expect_tx(&full[st], S::kKV);
        __syncwarp();
        if (has_box) tma_load_2d(ring + st * S::kKV + a * (kN * 128) + c * R * 128, map, a * 64, y, &full[st]);
        PA_TR(is_k ? kEvKIssued : kEvVIssued, j);
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------- MMA ---------------------------------
    bool ok = n_tiles == 0 || wait_all(q_full, 0);
    // PV of tile k: O += P V, P read from TMEM over the S columns of buffer k & 1.
    auto issue_pv = [&](int k) -> bool {
      const int st = k % kStagesV;
      if (!wait_all(&v_full[st], (k / kStagesV) & 1)) return false;
      PA_TR(kEvMmaVFull, k);
      // V rows past the context inside the last page chunk hold whatever the
      // pool holds there; P is 0 for them but 0 * NaN is NaN, so zero them.
      const int R = p.chunk_rows;
      const int z0 = L - (key0 + k * kN);
      if (z0 > 0 && z0 < kN && (L % R) != 0) {
        const int z1 = min(kN, ((L + R - 1) / R) * R - (key0 + k * kN));
        const int n16 = (z1 - z0) * KA * 8;  // 16-byte pieces
        for (int e = lane; e < n16; e += 32) {
          const int row = z0 + e / (KA * 8), rest = e % (KA * 8);
          const int a = rest / 8, c = rest % 8;
          uint4* dst = reinterpret_cast<uint4*>(smem + S::oV + st * S::kKV + a * (kN * 128) + row * 128 + c * 16);
          *dst = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (!wait_all(&p_full[k & 1], (k >> 1) & 1)) return false;
      PA_TR(kEvMmaP0, k);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t tP = (k & 1) ? tS1 : tS0;  // P (16-bit, two per column) over the first kN/2 columns
#pragma unroll
        for (int kk = 0; kk < KP; ++kk) {
          const uint64_t bd = sw128_desc(sV + st * S::kKV + kk * 2048, (kN * 128) >> 4, 64);
          tc_mma_ts(tO, tP + kk * 8, bd, kIdescO, (k > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&o_done[k & 1]);
#if !PA_TC_SLOT_BY_COMPLETION
        tc_commit(&v_empty[st]);
#endif
      }
      __syncwarp();
      PA_TR(kEvMmaPVIssued, k);
      return true;
    };
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int st = j % kStagesK;
      ok = wait_all(&k_full[st], (j / kStagesK) & 1);
      if (!ok) break;
      PA_TR(kEvMmaKFull, j);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t tS = (j & 1) ? tS1 : tS0;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint32_t koff = (ks / 4) * (kM * 128) + (ks % 4) * 32;
          const uint32_t kkoff = (ks / 4) * (kN * 128) + (ks % 4) * 32;
          const uint64_t ad = sw128_desc(sQ + koff, 1, 64);
          const uint64_t bd = sw128_desc(sK + st * S::kKV + kkoff, 1, 64);
          tc_mma(tS, ad, bd, kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[j & 1]);
#if !PA_TC_SLOT_BY_COMPLETION
        tc_commit(&k_empty[st]);
#endif
      }
      __syncwarp();
      PA_TR(kEvMmaSIssued, j);
      if (j > 0) ok = issue_pv(j - 1);
    }
    if (ok && n_tiles > 0) ok = issue_pv(n_tiles - 1);
    if (!ok && lane == 0) set_error(p.err, PA_DEVERR_WAIT);
  } else {
    // ------------------------------ softmax -------------------------------
    // Warp w owns rows 32w..32w+31 (its TMEM lanes) and all kN keys of every
    // tile: one online-softmax stream per row, running max and sum in
    // registers, O in TMEM.
    const int r = warp * 32 + lane;            // row = TMEM lane
    const int i = i0 + r / G, g = r % G;
    const int pos = prefix_mode ? L - 1 : L - C + i;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const uint32_t tOw = tO + lane_off;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!wait_all(&s_full[j & 1], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      if (warp < 2) PA_TR(warp ? kEvSm4SFull : kEvSm0SFull, j);
      tc_fence_after();
      float v[kN];
      {
        const uint32_t tS = ((j & 1) ? tS1 : tS0) + lane_off;
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc) tmem_ld32(tS + cc * 32, v + cc * 32);
        tmem_wait_ld();
      }
      const int t0 = key0 + j * kN;            // first key of the tile
      if (t0 + kN - 1 > pos_lo) {              // causal mask on the diagonal
#pragma unroll
        for (int e = 0; e < kN; ++e)
          if (t0 + e > pos) v[e] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = v[k];
#pragma unroll
      for (int e = 8; e < kN; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], v[e]);
#pragma unroll
      for (int k = 0; k < 4; ++k) mx8[k] = fmaxf(mx8[k], mx8[k + 4]);
      const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3]));
      const float m_tile = mx * p.scale_log2;
      const float m_new = fmaxf(m, m_tile);
      // Rescale only when the max grows by more than 2^8 (or on the first
      // finite max); otherwise keep the stale max, which bounds p by 2^8.
      const bool rescale = (m == -INFINITY) || (m_new > m + kRescaleLog2);
      const float m_use = rescale ? m_new : m;
      const float m_sub = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = exp2f(m - m_sub);    // 0 while nothing was seen yet
      const float2 ms2 = make_float2(-m_sub, -m_sub);
      uint32_t pk[kN / 2];
      float2 ps2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ps2[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < kN; e += 2) {
        const float2 x = __ffma2_rn(make_float2(v[e], v[e + 1]), sc2, ms2);
        const bool fma_path = ((e / 2) % 4) < PA_TC_POLY_OF_4;
        const uint32_t u = fma_path ? Fmt<T>::pack(ex2_sel<true>(x.x), ex2_sel<true>(x.y))
                                    : Fmt<T>::pack(ex2_sel<false>(x.x), ex2_sel<false>(x.y));
        pk[e / 2] = u;
        ps2[(e / 2) & 3] = __fadd2_rn(ps2[(e / 2) & 3], Fmt<T>::unpack2(u));  // sum of the rounded P
      }
      const float2 pa2 = __fadd2_rn(__fadd2_rn(ps2[0], ps2[1]), __fadd2_rn(ps2[2], ps2[3]));
      l = l * alpha + (pa2.x + pa2.y);
      m = m_use;
      // P goes back into TMEM over the first kN/2 columns of the S values this
      // warp just read (S buffer j&1; PV(j-2), the last reader of that buffer,
      // was issued before S(j), and tcgen05 MMAs run in issue order).
      {
        const uint32_t tP = ((j & 1) ? tS1 : tS0) + lane_off;
        tmem_st32(tP, reinterpret_cast<const float*>(pk));
      }
      if (j > 0) {
        // tcgen05.ld/st are warp-collective: the whole warp takes this branch
        // when any of its rows needs a rescale (the others multiply by 1). O
        // may be touched only once PV(j-1) is done.
        const bool need = rescale && alpha != 1.f;
        if (__any_sync(0xffffffffu, need)) {
          if (!wait_all(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
            tmem_wait_st();
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = need ? alpha : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            tmem_ld32(tOw + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= f;
            tmem_st32(tOw + cc * 32, o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
      if (warp < 2) PA_TR(warp ? kEvSm4PStored : kEvSm0PStored, j);
    }
    // epilogue: out = O / l (prefix mode: the unnormalised partial state)
    bool got = ok;
    if (ok && n_tiles > 0) {
      got = wait_all(&o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
      tc_fence_after();
    }
    if (!got) {
      if (lane == 0) set_error(p.err, PA_DEVERR_WAIT);
    } else {
      const float inv = (l > 0.f && n_tiles > 0) ? 1.f / l : 0.f;
      // Every thread reads its O row (warp-collective tcgen05.ld); only rows
      // of real queries (i < C) are stored.
      const bool store = i < C;
      T* orow = static_cast<T*>(p.out) + ((static_cast<int64_t>(b) * C + (store ? i : 0)) * p.num_q_heads + kvh * G + g) * D;
      // prefix mode: partial state of row (sequence i, head kvh*G + g), slot `split`
      const int64_t prow = (static_cast<int64_t>(store ? i : 0) * p.num_q_heads + kvh * G + g) * p.part_np + split;
      if (prefix_mode && store) {
        p.part_m[prow] = (l > 0.f && n_tiles > 0) ? m * 0.6931471805599453f : -INFINITY;
        p.part_l[prow] = n_tiles > 0 ? l : 0.f;
      }
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        if (n_tiles > 0) {
          tmem_ld32(tOw + cc * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
        if (!store) continue;
        if (prefix_mode) {  // unnormalised: sum_t 2^(s_t - m) v_t
          float* dst = p.part_o + prow * D + cc * 32;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
          continue;
        }
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w = make_uint4(Fmt<T>::pack_any(o[e] * inv, o[e + 1] * inv), Fmt<T>::pack_any(o[e + 2] * inv, o[e + 3] * inv),
                               Fmt<T>::pack_any(o[e + 4] * inv, o[e + 5] * inv), Fmt<T>::pack_any(o[e + 6] * inv, o[e + 7] * inv));
          *reinterpret_cast<uint4*>(orow + cc * 32 + e) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

template <typename T, int D, int G>
int launch(const Params& prm, const void* q, const void* k_cache, const void* v_cache, long long pool_rows,
           cudaStream_t stream) {
  constexpr int QT = kM / G;
  auto enc = encode_fn();
  if (!enc) return record_cuda_error(cudaErrorNotSupported, "prefill: cuTensorMapEncodeTiled unavailable");
  const CUtensorMapDataType dt =
      Fmt<T>::kCode == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap mq, mk, mv;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(prm.num_q_heads),
                                static_cast<cuuint64_t>(prm.num_seqs) * prm.chunk};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(prm.num_q_heads) * D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(QT)};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&mq, dt, 3, const_cast<void*>(q), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return record_cuda_error(cudaErrorInvalidValue, "prefill: encode q tensor map");
  }
  const cuuint64_t kdims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(pool_rows)};
  const cuuint64_t kstr[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t kbox[2] = {64, static_cast<cuuint32_t>(prm.chunk_rows)};
  const cuuint32_t kes[2] = {1, 1};
  if (enc(&mk, dt, 2, const_cast<void*>(k_cache), kdims, kstr, kbox, kes, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return record_cuda_error(cudaErrorInvalidValue, "prefill: encode k tensor map");
  if (enc(&mv, dt, 2, const_cast<void*>(v_cache), kdims, kstr, kbox, kes, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return record_cuda_error(cudaErrorInvalidValue, "prefill: encode v tensor map");

  auto kern = prefill_tc_kernel<T, D, G>;
  // At least a third of the SM's shared memory, so that at most two CTAs
  // (two TMEM allocations of 256 columns) share an SM.
  const int smem = Smem<D>::kAlloc > 78 * 1024 ? Smem<D>::kAlloc : 78 * 1024;
  // The attribute lives in the context: set it again after a device reset.
  static ContextCached<bool> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev].valid()) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return record_cuda_error(e, "prefill: set max dynamic shared memory");
    if (dev >= 0 && dev < 64) attr_done[dev].set(true);
  }
  dim3 grid((prm.chunk + QT - 1) / QT, prm.num_kv_heads, prm.prefix_len > 0 ? prm.key_splits : prm.num_seqs);
  kern<<<grid, kThreads, smem, stream>>>(mq, mk, mv, prm);
  return launch_status();
}

template <typename T, int D>
int by_group(const Params& prm, int G, const void* q, const void* k, const void* v, long long rows, cudaStream_t s) {
  switch (G) {
    case 1: return launch<T, D, 1>(prm, q, k, v, rows, s);
    case 2: return launch<T, D, 2>(prm, q, k, v, rows, s);
    case 4: return launch<T, D, 4>(prm, q, k, v, rows, s);
    case 8: return launch<T, D, 8>(prm, q, k, v, rows, s);
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace tc

int prefill_tcgen05(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int chunk_len,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                    pa_dtype dtype, cudaStream_t stream, const PrefixPartials* pp) {
  const long long pool_rows = static_cast<long long>(num_blocks) * num_kv_heads * block_size;
  if (pool_rows + 16 > 0x7fffffffLL || static_cast<long long>(num_seqs) * chunk_len > 0x7fffffffLL)
    return PA_ERR_SHAPE;
  if ((out && !aligned16(out)) || (reinterpret_cast<uintptr_t>(q) & 15)) return PA_ERR_ALIGN;
  tc::Params prm{};
  prm.out = out;
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
  prm.chunk_rows = block_size < 16 ? block_size : 16;
  prm.oob_row = static_cast<int>(pool_rows);  // first row past the pool: TMA reads zeros
  prm.scale_log2 = scale * tc::kLog2e;
  prm.trace = trace_buffer();
  if (pp) {
    prm.prefix_len = pp->prefix_len;
    prm.part_o = pp->part_o;
    prm.part_m = pp->part_m;
    prm.part_l = pp->part_l;
    prm.part_np = pp->num_partitions;
    prm.key_splits = pp->key_splits > 0 ? pp->key_splits : 1;
  }
  const int G = num_q_heads / num_kv_heads;
  if (dtype == PA_BF16) {
    if (head_dim == 128) return tc::by_group<__nv_bfloat16, 128>(prm, G, q, k_cache, v_cache, pool_rows, stream);
    if (head_dim == 64) return tc::by_group<__nv_bfloat16, 64>(prm, G, q, k_cache, v_cache, pool_rows, stream);
  } else if (dtype == PA_F16) {
    if (head_dim == 128) return tc::by_group<__half, 128>(prm, G, q, k_cache, v_cache, pool_rows, stream);
    if (head_dim == 64) return tc::by_group<__half, 64>(prm, G, q, k_cache, v_cache, pool_rows, stream);
  }
  return PA_ERR_UNSUPPORTED;
}

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
  return prefill_tcgen05(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                         chunk_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                         (cudaStream_t)stream, nullptr);
}
