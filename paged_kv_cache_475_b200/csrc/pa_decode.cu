// Paged decode attention on CUDA cores: pa_decode, pa_decode_splitkv and the
// split-KV / shared-prefix paths (their merge step is in pa_merge.cu).
//
// What it computes: out = softmax(scale * q K^T) V for one query token per
// sequence ("FlashAttention y PagedAttention", "Por qué la atención sale
// cara"), with K/V read page by page through the block table (same page,
// PagedAttention "Cómo funciona" step 5; "Cómo PagedAttention y RadixAttention
// optimizan el manejo del KV cache en LLMs", step 2) and the softmax kept
// online as a running max and running sum (FlashAttention "Cómo funciona").
// Split-KV evaluates the per-partition sums of eq. (4) of "Flash Attention vs
// Paged Attention" (算法原理) and pa_merge (pa_merge.cu) combines them.
//
// Design (B200, HBM-bound, no tensor cores):
//  * one CTA per (sequence, KV head[, partition]); every K/V page is read once
//    for all G = Hq/Hkv query heads of the group;
//  * each warp owns a private ring of STAGES shared-memory stages; lane 0
//    fills a stage with 1-D bulk copies (cp.async.bulk, TMA engine, no
//    multicast) of one 16-token tile of K and of V straight out of the page
//    that holds it, completing on the stage's mbarrier; block ids for the
//    warp's next 32 tiles are prefetched into registers one chunk ahead;
//  * scores: 8 (or 16) lanes split the head dim of one token, each lane keeps
//    4 (or 8) tokens x G heads of partial dots in packed-fp32 FMAs, and a
//    reduce-scatter over the lanes leaves every lane a few finished scores;
//  * online softmax in the log2 domain (q pre-scaled by scale*log2(e)),
//    probabilities through a 16 x G shared-memory slot, then P.V with each
//    lane owning D/32 output dims for all G heads;
//  * the warps' (m, l, o) states merge in shared memory at the end.
#include <mutex>
#include <type_traits>

#include "pa_common.cuh"

namespace pa {

constexpr int kTile = 16;              // tokens per pipeline stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T, int D, int G>
struct DecodeShape {
  static constexpr int kEsz = static_cast<int>(sizeof(T));
  static constexpr int kEpc = 16 / kEsz;                 // elements per 16-byte chunk
  static constexpr int kRowChunks = D / kEpc;            // 16-byte chunks per row
  static constexpr int kDGwant = (G >= 8) ? 16 : 8;
  static constexpr int kDG = kDGwant < kRowChunks ? kDGwant : kRowChunks;  // lanes per token (dims split)
  static constexpr int kTG = 32 / kDG;                   // token groups per warp
  static constexpr int kTPL = kTile / kTG;               // tokens per lane, score phase
  static constexpr int kCPL = kRowChunks / kDG;          // chunks per lane per token
  static constexpr int kQPL = kCPL * kEpc;               // q values per lane per head
  static constexpr int kNV = kTPL * G;                   // partial scores per lane
  static constexpr int kNF = kNV >= kDG ? kNV / kDG : 1; // finished scores per lane
  static constexpr int kDPL = D / 32;                    // output dims per lane, P.V phase
  static constexpr int kTileBytes = kTile * D * kEsz;    // one K (or V) tile
  static_assert(kCPL >= 1 && kQPL % 2 == 0, "head dim too small for the lane split");
  static_assert(kDPL % 2 == 0, "D must be a multiple of 64");
};

struct DecodeParams {
  void* out;                 // [N, Hq, D] (pa_decode)
  float* part_o;             // [N, Hq, NP, D] (split)
  float* part_m;             // [N, Hq, NP]
  float* part_l;             // [N, Hq, NP]
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  unsigned int* err;
  int max_blocks;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int partition;             // tokens per partition; 0 = whole sequence
  int num_parts;
  int longest_first;         // map CTA z-index r by longest-class-first order
  // Row pairing (single pass only; 0: off): CTAs with z >= pair_from take two
  // rows, ranks pair_from + 2 (z - pair_from) and the next one, two warps each.
  int pair_from;
  float q_scale;             // scale * log2(e)
  const void* k_new;         // fused append: [N, Hkv, D] rows of each sequence's newest token, or null
  const void* v_new;
  int skip_part0_seqs;       // split mode: partition 0 of sequences below this is computed elsewhere
  // Shared-prefix cascade (single pass, cascade_prefix > 0): sequences below
  // cascade_group start at token cascade_prefix and write partials into slot
  // cascade_slot of [N, Hq, num_parts, D]; the others write their rows to out.
  int cascade_prefix;
  int cascade_group;
  int cascade_slot;
  TraceRecord* trace;        // timeline records (PA_TRACE builds), else null
  // Read by the self-test instantiation only: copy-wait limit in SM cycles
  // and, with starve_first_copy set, warp 0 of CTA (0, 0, 0) arms its first
  // stage for a tile whose copies it never issues, so that wait must run out.
  long long wait_cycles;
  int starve_first_copy;
};

#ifndef PA_DECODE_CLASS_BITS
#define PA_DECODE_CLASS_BITS 2  // classes per octave of work: 2^bits
#endif
constexpr int kClassBits = PA_DECODE_CLASS_BITS;
constexpr int kNumClasses = 32 << kClassBits;   // 128 (bits = 2) or 256 (bits = 3)
constexpr int kClassesPerLane = kNumClasses / 32;

// Work class of a sequence with work w: 2^bits * floor(log2 w) plus the
// `bits` bits after the leading one (0 for w <= 0). Non-decreasing in w, so
// classes split the lengths into 2^bits geometric bands per octave.
__device__ inline int work_class(int w) {
  if (w <= 0) return 0;
  const unsigned u = static_cast<unsigned>(w);
  const int e = 31 - __clz(u);
  const unsigned mask = (1u << kClassBits) - 1u;
  const unsigned m = e >= kClassBits ? (u >> (e - kClassBits)) & mask : (u << (kClassBits - e)) & mask;
  return (e << kClassBits) + static_cast<int>(m);
}

// Sequences of ranks r0 and r1 (r1 < 0: none) in this order: classes in
// descending order, the sequences of one class by index; -1 for a rank
// outside [0, n). CTAs are dispatched in z order, so the
// longest contexts start first and short ones fill the tail (greedy
// longest-processing-time scheduling, to within one class). Work of sequence
// j is its length minus `skip` tokens when j < group. A counting sort: a
// shared-memory histogram of the classes, one warp's scan of it to find the
// class holding rank r and r's offset in it, then one warp's ballot walk
// over the class bytes for that offset; three CTA barriers in all (an exact
// bitonic sort of 256 keys takes 36, which on a batch of short sequences
// cost a fifth of the step). `scratch` (the copy ring, not yet in use)
// holds the counters, the answer and one class byte per sequence.
template <bool kTwo>
__device__ inline void longest_class_first_seqs(const int32_t* lens, int n, int r0, int r1, int* scratch, int group,
                                                int skip, int* b0, int* b1) {
  int* cnt = scratch;                                                                // [kNumClasses]
  int* answer = scratch + kNumClasses;                                               // [2]
  unsigned char* cls = reinterpret_cast<unsigned char*>(scratch + kNumClasses + 2);  // [n]
  for (int i = threadIdx.x; i < kNumClasses; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const int c = work_class(lens[j] - (j < group ? skip : 0));
    cls[j] = static_cast<unsigned char>(c);
    atomicAdd(&cnt[c], 1);
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // lane l owns classes top - i, i = 0 .. kClassesPerLane - 1 (descending)
    const int top = kNumClasses - 1 - kClassesPerLane * lane;
    int c_own[kClassesPerLane], tot = 0;
#pragma unroll
    for (int i = 0; i < kClassesPerLane; ++i) {
      c_own[i] = cnt[top - i];
      tot += c_own[i];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int start0 = incl - tot;  // sequences in the classes above this lane's
    for (int t = 0; t < (kTwo ? 2 : 1); ++t) {
      const int r = t ? r1 : r0;
      if (lane == 0) answer[t] = -1;  // no rank (r < 0 or r >= n): an empty row slot
      __syncwarp();
      if (r < 0 || r >= n) continue;
      int my_cls = -1, my_off = 0;
      int st = start0;
#pragma unroll
      for (int i = 0; i < kClassesPerLane; ++i) {
        if (r >= st && r < st + c_own[i]) {
          my_cls = top - i;
          my_off = r - st;
        }
        st += c_own[i];
      }
      const unsigned who = __ballot_sync(0xffffffffu, my_cls >= 0);  // one lane, as 0 <= r < n
      const int src = who ? __ffs(who) - 1 : 0;
      const int want = __shfl_sync(0xffffffffu, my_cls, src);
      int k = __shfl_sync(0xffffffffu, my_off, src);
      for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        const bool in = j < n && cls[j] == want;
        const unsigned m = __ballot_sync(0xffffffffu, in);
        const int c = __popc(m);
        if (k < c) {
          if (in && __popc(m & ((1u << lane) - 1u)) == k) answer[t] = j;
          break;
        }
        k -= c;
      }
    }
  }
  __syncthreads();
  *b0 = answer[0];
  *b1 = kTwo ? answer[1] : -1;
  __syncthreads();  // the staging area is the copy ring, which the caller fills next
}

// Reduce-scatter of a[NV] over the kDG lanes of a token group (xor offsets
// kDG/2 .. 1): at each level a lane keeps one half of its values and adds the
// partner's copy of that half. Levels past a single value all-reduce.
template <int NV, int OFF>
struct ReduceScatter {
  __device__ static inline void run(float* a, int lane) {
    if constexpr (OFF >= 1) {
      if constexpr (NV >= 2) {
        constexpr int H = NV / 2;
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = upper ? a[i] : a[H + i];
          const float keep = upper ? a[H + i] : a[i];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
        }
        ReduceScatter<H, OFF / 2>::run(a, lane);
      } else {
        a[0] += __shfl_xor_sync(0xffffffffu, a[0], OFF);
        ReduceScatter<1, OFF / 2>::run(a, lane);
      }
    }
  }
};

// Index (into the original a[]) of a lane's first finished value.
template <int NV, int DG>
__device__ inline int scatter_base(int lane) {
  int base = 0, n = NV;
#pragma unroll
  for (int off = DG / 2; off >= 1; off /= 2) {
    if (n >= 2) {
      n /= 2;
      if (lane & off) base += n;
    }
  }
  return base;
}

// Does xor offset `off` connect two lanes holding different tokens of the same
// head (as opposed to different heads, or copies of the same value)?
template <int NV, int DG, int TPL>
__host__ __device__ constexpr bool same_head_offset(int off) {
  if (off >= DG) return true;  // token-group bits
  int n = NV;
  for (int o = DG / 2; o >= 1; o /= 2) {
    if (n >= 2) {
      n /= 2;
      if (o == off) return n < TPL;
    } else if (o == off) {
      return false;  // all-reduce level: both lanes hold the same value
    }
  }
  return false;
}

template <int NV, int DG, int TPL, typename Op>
__device__ inline float head_reduce(float v, Op op) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2)
    if (same_head_offset<NV, DG, TPL>(off)) v = op(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Lane (token group 0) that holds head g's first finished value.
template <int NV, int DG, int TPL>
__device__ inline int head_src_lane(int g) {
  const int base = g * TPL;
  int lane = 0, n = NV;
#pragma unroll
  for (int off = DG / 2; off >= 1; off /= 2) {
    if (n >= 2) {
      n /= 2;
      if (base & n) lane |= off;
    }
  }
  return lane;
}

struct MaxOp { __device__ float operator()(float a, float b) const { return fmax_nan(a, b); } };
struct SumOp { __device__ float operator()(float a, float b) const { return a + b; } };

template <typename T, int D, int G, int NW, int STAGES>
struct DecodeSmem {
  using S = DecodeShape<T, D, G>;
  static constexpr int kStageBytes = 2 * S::kTileBytes;
  static constexpr int kRingBytes = NW * STAGES * kStageBytes;
  static constexpr int kProbBytes = NW * kTile * G * 4;
  static constexpr int kMergeBytes = NW * G * (D + 2) * 4;
  static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kBarOff = kDataBytes + kProbBytes;
  static constexpr int kValidOff = kBarOff + NW * STAGES * 8;
  static constexpr int kTotal = kValidOff + NW * STAGES * 4 + 16;
};

// No minimum-blocks bound: the fp16 / bf16 kernels at D = 128 fit three CTAs
// per SM (167 registers, 67 KB) without one, and capping the registers at 170
// to force it made the compiler trade ILP for registers (2.5% slower).
template <typename T, int D, int G, int NW, int STAGES, bool kSelfTest = false, bool kPaired = false>
__global__ void __launch_bounds__(NW * 32, 1)
decode_kernel(const DecodeParams p) {
  using S = DecodeShape<T, D, G>;
  using M = DecodeSmem<T, D, G, NW, STAGES>;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int part = blockIdx.x;
  const int kvh = blockIdx.y;
  const bool split = p.partition > 0;
#if PA_TRACE
  const unsigned long long tr_start = global_ns();
  unsigned long long tr_first = 0;
#endif
  // A shared prefix's partition was computed once for its whole group; a
  // group member must reach past the prefix (its newest token is its own).
  if (split && part == 0 && static_cast<int>(blockIdx.z) < p.skip_part0_seqs) {
    if (threadIdx.x == 0 && kvh == 0 && p.context_lens[blockIdx.z] <= p.partition) set_error(p.err, PA_DEVERR_CONTEXT);
    return;
  }
  // Rows of this CTA: one, or two short ones (ranks past the longest
  // pair_from) with NW/2 warps each. Warp `warp` works on row `sub` as warp
  // `wr` of the row's `wpr`; a row slot past the batch (b < 0) is empty.
  const int z = static_cast<int>(blockIdx.z);
  // Pairing is a separate instantiation (kPaired), so that every other
  // launch keeps the fixed one-row layout (its divisions by constants, its
  // unrolled merge); a paired launch's first pair_from CTAs take one row.
  const bool paired = kPaired && !split && p.pair_from > 0 && z >= p.pair_from;
  const int wpr = paired ? NW / 2 : NW;
  const int sub = warp / wpr;
  const int wr = warp - sub * wpr;
  const int r0 = paired ? p.pair_from + 2 * (z - p.pair_from) : z;
  const int r1 = paired ? r0 + 1 : -1;
  int b_row0, b_row1;
  if (p.longest_first) {
    longest_class_first_seqs<kPaired>(p.context_lens, p.num_seqs, r0, r1, reinterpret_cast<int*>(smem),
                                      p.cascade_group, p.cascade_prefix, &b_row0, &b_row1);
  } else {
    b_row0 = r0 < p.num_seqs ? r0 : -1;
    b_row1 = (r1 >= 0 && r1 < p.num_seqs) ? r1 : -1;
  }
  const int b = sub ? b_row1 : b_row0;
  const bool row_lead = wr == 0 && lane == 0;  // reports this row's errors
  const bool cascade_member = p.cascade_prefix > 0 && b >= 0 && b < p.cascade_group;
  if (cascade_member && row_lead && kvh == 0 && p.context_lens[b] <= p.cascade_prefix)
    set_error(p.err, PA_DEVERR_CONTEXT);

  // ---- context range of this warp's row --------------------------------------
  int L = b >= 0 ? p.context_lens[b] : 0;
  if (L < 0 || L > p.max_blocks * p.block_size) {
    if (row_lead) set_error(p.err, PA_DEVERR_CONTEXT);
    L = L < 0 ? 0 : p.max_blocks * p.block_size;
  }
  if (split && part == p.num_parts - 1 && L > p.num_parts * p.partition && threadIdx.x == 0)
    set_error(p.err, PA_DEVERR_CONTEXT);
  const int t_begin = split ? part * p.partition : (cascade_member ? p.cascade_prefix : 0);
  int t_end = split ? min(L, t_begin + p.partition) : L;
  if (t_end < t_begin) t_end = t_begin;
  const int n_tiles = (t_end - t_begin + kTile - 1) / kTile;
  const int my_tiles = wr < n_tiles ? (n_tiles - wr + wpr - 1) / wpr : 0;

  unsigned char* ring = smem + warp * STAGES * M::kStageBytes;
  float* prob = reinterpret_cast<float*>(smem + M::kDataBytes) + warp * kTile * G;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + M::kBarOff) + warp * STAGES;
  int* stage_valid = reinterpret_cast<int*>(smem + M::kValidOff) + warp * STAGES;

  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const T* kc = static_cast<const T*>(p.k_cache);
  const T* vc = static_cast<const T*>(p.v_cache);
  const int32_t* bt = p.block_tables + static_cast<int64_t>(b < 0 ? 0 : b) * p.max_blocks;
  const int B = p.block_size;
  const int n_seq_blocks = (L + B - 1) / B;

  const uint64_t policy = l2_evict_first_policy();

  // Block ids of this warp's tiles k = 32*c + lane (two ids per tile when B = 8).
  auto load_ids = [&](int chunk, int& id0, int& id1) {
    const int k = chunk * 32 + lane;
    id0 = -1;
    id1 = -1;
    if (k < my_tiles) {
      const int t0 = t_begin + (wr + wpr * k) * kTile;
      const int j = t0 / B;
      id0 = bt[j];
      if (B < kTile && j + 1 < n_seq_blocks && t0 + B < t_end) id1 = bt[j + 1];
    }
  };
  int cur0, cur1, nxt0, nxt1;
  load_ids(0, cur0, cur1);
  load_ids(1, nxt0, nxt1);
  int ids_chunk = 0;

  // Self-test instantiations only (a template flag, so that the attention
  // kernels carry neither the check nor the limit in registers).
  const bool starve = kSelfTest && p.starve_first_copy && warp == 0 && blockIdx.x == 0 && blockIdx.y == 0 &&
                      blockIdx.z == 0;
  const long long wait_limit = kSelfTest ? p.wait_cycles : 4000000000LL;

  // Issue the copies of tile k into stage k % STAGES (all lanes call; lane 0 copies).
  auto issue = [&](int k) {
    const int chunk = k >> 5;
    if (chunk != ids_chunk) {  // advance the prefetched id window
      cur0 = nxt0;
      cur1 = nxt1;
      ids_chunk = chunk;
      load_ids(chunk + 1, nxt0, nxt1);
    }
    const int id0 = __shfl_sync(0xffffffffu, cur0, k & 31);
    const int id1 = __shfl_sync(0xffffffffu, cur1, k & 31);
    if (lane == 0) {
      const int s = k % STAGES;
      const int t0 = t_begin + (wr + wpr * k) * kTile;
      const int nvalid = min(kTile, t_end - t0);
      unsigned char* kdst = ring + s * M::kStageBytes;
      unsigned char* vdst = kdst + S::kTileBytes;
      // Validate every block id before any copy; a bad id skips the tile.
      bool ok;
      const bool second = B < kTile && nvalid > B;
      if (B >= kTile) {
        ok = id0 >= 0 && id0 < p.num_blocks;
      } else {
        ok = id0 >= 0 && id0 < p.num_blocks && (!second || (id1 >= 0 && id1 < p.num_blocks));
      }
      // The stage's valid-token count is written before the arrive (release),
      // so the lanes that acquire the completed phase see it.
      stage_valid[s] = ok ? nvalid : 0;
      if (!ok) {
        set_error(p.err, PA_DEVERR_BLOCK_ID);
        mbar_arrive_expect_tx(&bars[s], 0);
      } else if (starve && k == 0) {
        mbar_arrive_expect_tx(&bars[s], 2u * S::kTileBytes);  // no copy follows: the wait must time out
      } else if (B >= kTile) {
        const int64_t off = ((static_cast<int64_t>(id0) * p.num_kv_heads + kvh) * B + (t0 % B)) * D;
        mbar_arrive_expect_tx(&bars[s], 2u * S::kTileBytes);
        bulk_g2s(kdst, kc + off, S::kTileBytes, &bars[s], policy);
        bulk_g2s(vdst, vc + off, S::kTileBytes, &bars[s], policy);
      } else {  // B == 8: two half tiles, the second only if it holds a valid token
        const uint32_t half = S::kTileBytes / 2;
        mbar_arrive_expect_tx(&bars[s], (second ? 2u : 1u) * 2u * half);
        const int64_t off0 = (static_cast<int64_t>(id0) * p.num_kv_heads + kvh) * B * D;
        bulk_g2s(kdst, kc + off0, half, &bars[s], policy);
        bulk_g2s(vdst, vc + off0, half, &bars[s], policy);
        if (second) {
          const int64_t off1 = (static_cast<int64_t>(id1) * p.num_kv_heads + kvh) * B * D;
          bulk_g2s(kdst + half, kc + off1, half, &bars[s], policy);
          bulk_g2s(vdst + half, vc + off1, half, &bars[s], policy);
        }
      }
    }
  };

  // ---- q for this lane: G heads x kQPL dims, pre-scaled ----------------------
  const int dg = lane % S::kDG;
  const int tg = lane / S::kDG;
  float2 q2[G][S::kQPL / 2];
  {
    const T* qb = static_cast<const T*>(p.q) + (static_cast<int64_t>(b < 0 ? 0 : b) * p.num_q_heads + kvh * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int c = 0; c < S::kCPL; ++c) {
        const int ci = c * S::kDG + dg;
        const uint4 u = *reinterpret_cast<const uint4*>(qb + g * D + ci * S::kEpc);
        float f[S::kEpc];
        unpack16(u, f, T());
#pragma unroll
        for (int e = 0; e < S::kEpc; e += 2)
          q2[g][(c * S::kEpc + e) / 2] = make_float2(f[e] * p.q_scale, f[e + 1] * p.q_scale);
      }
    }
  }

  // ---- running state ---------------------------------------------------------
  float m_run[G];
  float2 acc[G][S::kDPL / 2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
#pragma unroll
    for (int j = 0; j < S::kDPL / 2; ++j) acc[g][j] = make_float2(0.f, 0.f);
  }
  float l_part = 0.f;  // partial sum of this lane's own head, own tokens
  const int base_idx = scatter_base<S::kNV, S::kDG>(lane);
  const int my_head = base_idx / S::kTPL;

  // ---- fused append: the CTA whose range holds position L-1 writes the
  // sequence's newest K/V row (this KV head) into its slot before reading
  // it. Only the warp that owns the tile holding L-1 (tiles are dealt to
  // warps round-robin) writes it and only that warp ever reads it, so the
  // other warps start their copies at once. Generic stores, then the proxy
  // fence by every writing lane and a warp barrier, so that lane 0's bulk
  // copies (async proxy) see the row.
  if (p.k_new != nullptr && L > 0 && t_begin <= L - 1 && L - 1 < t_end &&
      wr == ((L - 1 - t_begin) / kTile) % wpr) {
    const int pos = L - 1;
    const int phys = bt[pos / B];
    if (phys >= 0 && phys < p.num_blocks) {
      constexpr int kChunks = D * S::kEsz / 16;  // 16-byte pieces of one row
      const int64_t src = (static_cast<int64_t>(b) * p.num_kv_heads + kvh) * D;
      const int64_t dst = ((static_cast<int64_t>(phys) * p.num_kv_heads + kvh) * B + pos % B) * D;
      for (int c = lane; c < 2 * kChunks; c += 32) {
        const bool is_v = c >= kChunks;
        const int cc = is_v ? c - kChunks : c;
        const uint4 val = reinterpret_cast<const uint4*>(static_cast<const T*>(is_v ? p.v_new : p.k_new) + src)[cc];
        reinterpret_cast<uint4*>(const_cast<T*>(is_v ? vc : kc) + dst)[cc] = val;
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");
    } else if (lane == 0) {
      set_error(p.err, PA_DEVERR_BLOCK_ID);
    }
    __syncwarp();
  }
  // ---- pipeline --------------------------------------------------------------
  const int prologue = my_tiles < STAGES ? my_tiles : STAGES;
  for (int k = 0; k < prologue; ++k) issue(k);
  __syncwarp();

  bool aborted = false;
  int k = 0;
  for (; k < my_tiles; ++k) {
    const int s = k % STAGES;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[s], (k / STAGES) & 1, wait_limit))) {
      if (lane == 0) set_error(p.err, PA_DEVERR_WAIT);
      aborted = true;
      break;
    }
#if PA_TRACE
    if (k == 0 && warp == 0) tr_first = global_ns();
#endif
    const int nvalid = stage_valid[s];
    const unsigned char* ktile = ring + s * M::kStageBytes;
    const unsigned char* vtile = ktile + S::kTileBytes;

    if (nvalid > 0) {
      // -- scores: partial dots over this lane's dims for its kTPL tokens --
      float a[S::kNV];
      {
        float2 part2[G][S::kTPL];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int i = 0; i < S::kTPL; ++i) part2[g][i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < S::kTPL; ++i) {
          const int t = tg + S::kTG * i;
#pragma unroll
          for (int c = 0; c < S::kCPL; ++c) {
            const int ci = c * S::kDG + dg;
            const uint4 u = *reinterpret_cast<const uint4*>(ktile + (t * S::kRowChunks + ci) * 16);
            float f[S::kEpc];
            unpack16(u, f, T());
#pragma unroll
            for (int e = 0; e < S::kEpc; e += 2) {
              const float2 kv = make_float2(f[e], f[e + 1]);
#pragma unroll
              for (int g = 0; g < G; ++g) part2[g][i] = ffma2(q2[g][(c * S::kEpc + e) / 2], kv, part2[g][i]);
            }
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int i = 0; i < S::kTPL; ++i) a[g * S::kTPL + i] = part2[g][i].x + part2[g][i].y;
      }
      ReduceScatter<S::kNV, S::kDG / 2>::run(a, lane);

      // -- mask and tile max per head --
      float vmax = -INFINITY;
#pragma unroll
      for (int f = 0; f < S::kNF; ++f) {
        const int idx = base_idx + f;
        const int t = tg + S::kTG * (idx % S::kTPL);
        if (t >= nvalid) a[f] = -INFINITY;
        vmax = fmax_nan(vmax, a[f]);
      }
      vmax = head_reduce<S::kNV, S::kDG, S::kTPL>(vmax, MaxOp());
      float alpha[G], m_use[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float tmax = __shfl_sync(0xffffffffu, vmax, head_src_lane<S::kNV, S::kDG, S::kTPL>(g));
        const float m_new = fmax_nan(m_run[g], tmax);
        m_use[g] = m_new == -INFINITY ? 0.f : m_new;
        alpha[g] = exp2f(m_run[g] - m_use[g]);  // exp2(-inf) = 0 on the first tile
        m_run[g] = m_new;
      }
      // -- probabilities of this lane's scores into the tile's prob slot --
      float psum = 0.f;
#pragma unroll
      for (int f = 0; f < S::kNF; ++f) {
        const int idx = base_idx + f;
        const int t = tg + S::kTG * (idx % S::kTPL);
        float mh = m_use[0];
#pragma unroll
        for (int g = 1; g < G; ++g) mh = (my_head == g) ? m_use[g] : mh;
        const float pr = exp2f(a[f] - mh);
        psum += pr;
        prob[t * G + my_head] = pr;
      }
      {
        float ah = alpha[0];
#pragma unroll
        for (int g = 1; g < G; ++g) ah = (my_head == g) ? alpha[g] : ah;
        l_part = l_part * ah + psum;
      }
      __syncwarp();

      // -- P.V: this lane's kDPL output dims for all G heads --
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < S::kDPL / 2; ++j) {
          acc[g][j].x *= alpha[g];
          acc[g][j].y *= alpha[g];
        }
      auto pv_token = [&](int t) {
        float vf[S::kDPL];
        const unsigned char* vrow = vtile + (t * D + lane * S::kDPL) * S::kEsz;
        if constexpr (S::kDPL * S::kEsz == 16) {
          unpack16(*reinterpret_cast<const uint4*>(vrow), vf, T());
        } else if constexpr (S::kDPL * S::kEsz == 8) {
          unpack8(*reinterpret_cast<const uint2*>(vrow), vf, T());
        } else {
          unpack4(*reinterpret_cast<const uint32_t*>(vrow), vf, T());
        }
        float pg[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g = 0; g < G; g += 4) {
            const float4 p4 = *reinterpret_cast<const float4*>(prob + t * G + g);
            pg[g] = p4.x; pg[g + 1] = p4.y; pg[g + 2] = p4.z; pg[g + 3] = p4.w;
          }
        } else if constexpr (G == 2) {
          const float2 p2 = *reinterpret_cast<const float2*>(prob + t * G);
          pg[0] = p2.x; pg[1] = p2.y;
        } else {
          pg[0] = prob[t];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 pp = make_float2(pg[g], pg[g]);
#pragma unroll
          for (int j = 0; j < S::kDPL / 2; ++j)
            acc[g][j] = ffma2(pp, make_float2(vf[2 * j], vf[2 * j + 1]), acc[g][j]);
        }
      };
      if (nvalid == kTile) {
#pragma unroll
        for (int t = 0; t < kTile; ++t) pv_token(t);
      } else {
        for (int t = 0; t < nvalid; ++t) pv_token(t);
      }
    }
    __syncwarp();
    if (k + STAGES < my_tiles) issue(k + STAGES);
  }

  if (aborted) {
    // Let this warp's copies still in flight land before the CTA exits.
    const int issued = my_tiles < k + STAGES ? my_tiles : k + STAGES;
    const long long drain_limit = kSelfTest ? p.wait_cycles : 400000000LL;
    for (int kk = k; kk < issued; ++kk) mbar_wait(&bars[kk % STAGES], (kk / STAGES) & 1, drain_limit);
  }

  // ---- per-warp finish: l for every head -------------------------------------
  const float l_head = head_reduce<S::kNV, S::kDG, S::kTPL>(l_part, SumOp());
  float l_run[G];
#pragma unroll
  for (int g = 0; g < G; ++g) l_run[g] = __shfl_sync(0xffffffffu, l_head, head_src_lane<S::kNV, S::kDG, S::kTPL>(g));

  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  float* mo = reinterpret_cast<float*>(smem);                   // [NW][G][D]
  float* mm = mo + NW * G * D;                                   // [NW][G]
  float* ml = mm + NW * G;                                       // [NW][G]
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int j = 0; j < S::kDPL / 2; ++j)
      *reinterpret_cast<float2*>(mo + (warp * G + g) * D + lane * S::kDPL + 2 * j) = acc[g][j];
    if (lane == 0) {
      mm[warp * G + g] = m_run[g];
      ml[warp * G + g] = l_run[g];
    }
  }
  __syncthreads();

  const int n_rows = paired ? 2 : 1;
  for (int i = threadIdx.x; i < n_rows * G * D; i += NW * 32) {
    const int rs = i / (G * D);  // row slot: its warps are rs * wpr .. rs * wpr + wpr - 1
    const int g = (i / D) % G, d = i % D;
    const int rb = rs ? b_row1 : b_row0;
    if (rb < 0) continue;
    const int w0 = rs * wpr;
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if (!kPaired || w < wpr) Mx = fmax_nan(Mx, mm[(w0 + w) * G + g]);
    float o = 0.f, l = 0.f;
    if (Mx != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) {
        if (kPaired && ww >= wpr) break;
        const int w = w0 + ww;
        const float mw = mm[w * G + g];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - Mx);
        o += sc * mo[(w * G + g) * D + d];
        l += sc * ml[w * G + g];
      }
    }
    const int h = kvh * G + g;
    const bool member = p.cascade_prefix > 0 && rb < p.cascade_group;
    if (split || member) {
      const int slot = split ? part : p.cascade_slot;
      const int64_t row = (static_cast<int64_t>(rb) * p.num_q_heads + h) * p.num_parts + slot;
      p.part_o[row * D + d] = o;
      if (d == 0) {
        p.part_m[row] = Mx == -INFINITY ? -INFINITY : Mx * kLn2;
        p.part_l[row] = l;
      }
    } else {
      T* out = static_cast<T*>(p.out) + (static_cast<int64_t>(rb) * p.num_q_heads + h) * D;
      out[d] = Elem<T>::from_f(!(l <= 0.f) ? o / l : 0.f);  // l = NaN passes NaN on
    }
  }
#if PA_TRACE
  if (threadIdx.x == 0) {
    const long long idx = blockIdx.x + static_cast<long long>(gridDim.x) * (blockIdx.y + static_cast<long long>(gridDim.y) * blockIdx.z);
    if (p.trace != nullptr && idx < kTraceMax)
      p.trace[idx] = TraceRecord{tr_start, tr_first, global_ns(), sm_id(), b, kvh, part, t_end - t_begin,
                                 split ? 1 : (cascade_member ? 2 : 0)};
  }
#endif
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif
#ifndef PA_DECODE_LPT_MAX_SEQS
#define PA_DECODE_LPT_MAX_SEQS 512  // class ordering stages n bytes + counters in the copy ring (>= 32 KB)
#endif
constexpr int kDecodeWarps = PA_DECODE_WARPS;
constexpr int kDecodeStages = PA_DECODE_STAGES;

template <typename T, int D, int G, bool kSelfTest = false, bool kPaired = false>
int launch_decode(const DecodeParams& prm, int grid_x, cudaStream_t stream) {
  constexpr int NW = kDecodeWarps;
  constexpr int ST = (DecodeShape<T, D, G>::kTileBytes >= 8192 && kDecodeStages > 2) ? 2 : kDecodeStages;
  using M = DecodeSmem<T, D, G, NW, ST>;
  auto kern = decode_kernel<T, D, G, NW, ST, kSelfTest, kPaired>;
  // The attribute lives in the context: set it again after a device reset.
  static ContextCached<bool> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev].valid()) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, M::kTotal);
    if (e != cudaSuccess) return record_cuda_error(e, "decode: set max dynamic shared memory");
    // all of the SM's unified L1/shared memory as shared memory, so that three CTAs fit
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return record_cuda_error(e, "decode: set the shared memory carveout");
    if (dev >= 0 && dev < 64) attr_done[dev].set(true);
  }
  const int grid_z = prm.pair_from > 0 ? prm.pair_from + (prm.num_seqs - prm.pair_from + 1) / 2 : prm.num_seqs;
  dim3 grid(grid_x, prm.num_kv_heads, grid_z);
  kern<<<grid, NW * 32, M::kTotal, stream>>>(prm);
  return launch_status();
}

template <typename T, int D>
int dispatch_group(const DecodeParams& prm, int G, int grid_x, cudaStream_t s) {
  // Paired launches exist for the 16-bit types (fp32 caches launch one row per CTA).
  if constexpr (!std::is_same<T, float>::value) {
    if (prm.pair_from > 0) {
      switch (G) {
        case 1: return launch_decode<T, D, 1, false, true>(prm, grid_x, s);
        case 2: return launch_decode<T, D, 2, false, true>(prm, grid_x, s);
        case 4: return launch_decode<T, D, 4, false, true>(prm, grid_x, s);
        case 8: return launch_decode<T, D, 8, false, true>(prm, grid_x, s);
      }
      return PA_ERR_UNSUPPORTED;
    }
  }
  DecodeParams one = prm;
  one.pair_from = 0;
  switch (G) {
    case 1: return launch_decode<T, D, 1>(one, grid_x, s);
    case 2: return launch_decode<T, D, 2>(one, grid_x, s);
    case 4: return launch_decode<T, D, 4>(one, grid_x, s);
    case 8: return launch_decode<T, D, 8>(one, grid_x, s);
  }
  return PA_ERR_UNSUPPORTED;
}

template <typename T>
int dispatch_dim(const DecodeParams& prm, int D, int G, int grid_x, cudaStream_t s) {
  if (D == 64) return dispatch_group<T, 64>(prm, G, grid_x, s);
  if (D == 128) return dispatch_group<T, 128>(prm, G, grid_x, s);
  return PA_ERR_UNSUPPORTED;
}

#ifndef PA_DECODE_PAIR_WAVES
#define PA_DECODE_PAIR_WAVES 3  // pair rows when one row per CTA would take more waves than this (0: never)
#endif
#ifndef PA_DECODE_PAIR_KEEP_DIV
#define PA_DECODE_PAIR_KEEP_DIV 8  // the longest num_seqs / this ranks keep a CTA each (4 and 2 measured slower)
#endif

// Rank from which a single-pass launch gives each CTA two rows (0: none).
// Only a batch whose one-row-per-CTA grid would take more than
// PA_DECODE_PAIR_WAVES waves of three CTAs per SM is paired: there the CTAs
// are short and their start-up (ordering, block ids, first copies) is a
// large share of their life, so two rows with two warps each per CTA keep
// twice as many rows in flight per SM. The longest num_seqs / KEEP_DIV
// ranks (the first CTAs in longest-class-first order) keep all four warps.
int decode_pair_from(int num_seqs, int num_kv_heads) {
  if (PA_DECODE_PAIR_WAVES <= 0 || num_seqs < 2) return 0;
  static int sms[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int n_sm = dev >= 0 && dev < 64 ? sms[dev] : 0;
  if (n_sm <= 0) {
    if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0) return 0;
    if (dev >= 0 && dev < 64) sms[dev] = n_sm;
  }
  const long long ctas = static_cast<long long>(num_seqs) * num_kv_heads;
  if (ctas <= static_cast<long long>(PA_DECODE_PAIR_WAVES) * 3 * n_sm) return 0;
  const int keep = num_seqs / PA_DECODE_PAIR_KEEP_DIV;
  return keep < 1 ? 1 : keep;
}

int run_decode(DecodeParams prm, int D, float scale, pa_dtype dt, int grid_x, cudaStream_t s) {
  const int G = prm.num_q_heads / prm.num_kv_heads;
  prm.q_scale = scale * kLog2e;
  prm.err = device_error_word();
  prm.trace = trace_buffer();
  switch (dt) {
    case PA_F32: return dispatch_dim<float>(prm, D, G, grid_x, s);
    case PA_F16: return dispatch_dim<__half>(prm, D, G, grid_x, s);
    case PA_BF16: return dispatch_dim<__nv_bfloat16>(prm, D, G, grid_x, s);
  }
  return PA_ERR_DTYPE;
}

int check_decode_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      int max_blocks, const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dt) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks < 0 || max_blocks < 0)
    return PA_ERR_SHAPE;
  if (dt != PA_F32 && dt != PA_F16 && dt != PA_BF16) return PA_ERR_DTYPE;
  if (num_q_heads % num_kv_heads) return PA_ERR_SHAPE;
  if (!supported_head_dim(head_dim) || !supported_block(block_size) ||
      !supported_group(num_q_heads / num_kv_heads))
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_ALIGN;
  return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" PA_API int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                                int head_dim, int block_size, int num_blocks, float scale, pa_dtype dtype,
                                void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!out) return PA_ERR_NULL;
  if (num_seqs > 65535) return PA_ERR_SHAPE;
  DecodeParams prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = 0;
  prm.num_parts = 1;
  prm.longest_first = num_seqs > 1 && num_seqs <= PA_DECODE_LPT_MAX_SEQS;
  prm.pair_from = decode_pair_from(num_seqs, num_kv_heads);
  return run_decode(prm, head_dim, scale, dtype, 1, (cudaStream_t)stream);
}

extern "C" PA_API int pa_decode_selftest_starved_wait(void* out, const void* q, const void* k_cache,
                                                      const void* v_cache, const int32_t* block_tables,
                                                      int max_blocks_per_seq, const int32_t* context_lens,
                                                      int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                      int block_size, int num_blocks, float scale, pa_dtype dtype,
                                                      long long wait_cycles, void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!out) return PA_ERR_NULL;
  if (num_seqs > 65535 || wait_cycles < 1000 || wait_cycles > 4000000000LL) return PA_ERR_SHAPE;
  DecodeParams prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = 0;
  prm.num_parts = 1;
  prm.longest_first = num_seqs > 1 && num_seqs <= PA_DECODE_LPT_MAX_SEQS;
  prm.pair_from = decode_pair_from(num_seqs, num_kv_heads);
  prm.wait_cycles = wait_cycles;
  prm.starve_first_copy = 1;
  if (dtype != PA_F16 || head_dim != 128) return PA_ERR_UNSUPPORTED;  // the one instantiation kept for it
  prm.q_scale = scale * kLog2e;
  prm.err = device_error_word();
  prm.trace = trace_buffer();
  cudaStream_t s = (cudaStream_t)stream;
  switch (num_q_heads / num_kv_heads) {
    case 1: return launch_decode<__half, 128, 1, true>(prm, 1, s);
    case 2: return launch_decode<__half, 128, 2, true>(prm, 1, s);
    case 4: return launch_decode<__half, 128, 4, true>(prm, 1, s);
    case 8: return launch_decode<__half, 128, 8, true>(prm, 1, s);
  }
  return PA_ERR_UNSUPPORTED;
}

extern "C" PA_API int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                                       void* k_cache, void* v_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                       int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                       int num_blocks, float scale, pa_dtype dtype, void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!out || !k_new || !v_new) return PA_ERR_NULL;
  if (!aligned16(k_new) || !aligned16(v_new)) return PA_ERR_ALIGN;
  if (num_seqs > 65535) return PA_ERR_SHAPE;
  DecodeParams prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.k_new = k_new;
  prm.v_new = v_new;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = 0;
  prm.num_parts = 1;
  prm.longest_first = num_seqs > 1 && num_seqs <= PA_DECODE_LPT_MAX_SEQS;
  return run_decode(prm, head_dim, scale, dtype, 1, (cudaStream_t)stream);
}

extern "C" PA_API int pa_decode_splitkv_append(float* part_o, float* part_m, float* part_l, const void* q,
                                               const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                               const int32_t* block_tables, int max_blocks_per_seq,
                                               const int32_t* context_lens, int num_seqs, int num_q_heads,
                                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                               int partition_size, int num_partitions, float scale, pa_dtype dtype,
                                               void* stream) {
  if (!k_new || !v_new) return PA_ERR_NULL;
  if (!aligned16(k_new) || !aligned16(v_new)) return PA_ERR_ALIGN;
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!part_o || !part_m || !part_l) return PA_ERR_NULL;
  if (!aligned16(part_o)) return PA_ERR_ALIGN;
  if (partition_size <= 0 || partition_size % kTile || num_partitions <= 0) return PA_ERR_WORKSPACE;
  if (num_seqs > 65535 || num_partitions > (1 << 30)) return PA_ERR_SHAPE;
  DecodeParams prm{};
  prm.part_o = part_o;
  prm.part_m = part_m;
  prm.part_l = part_l;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.k_new = k_new;
  prm.v_new = v_new;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = partition_size;
  prm.num_parts = num_partitions;
  return run_decode(prm, head_dim, scale, dtype, num_partitions, (cudaStream_t)stream);
}

extern "C" PA_API int pa_decode_splitkv(float* part_o, float* part_m, float* part_l, const void* q,
                                        const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                        int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                        int num_blocks, int partition_size, int num_partitions, float scale,
                                        pa_dtype dtype, void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!part_o || !part_m || !part_l) return PA_ERR_NULL;
  if (!aligned16(part_o)) return PA_ERR_ALIGN;
  if (partition_size <= 0 || partition_size % kTile || num_partitions <= 0) return PA_ERR_WORKSPACE;
  if (num_seqs > 65535 || num_partitions > (1 << 30)) return PA_ERR_SHAPE;
  DecodeParams prm{};
  prm.part_o = part_o;
  prm.part_m = part_m;
  prm.part_l = part_l;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = partition_size;
  prm.num_parts = num_partitions;
  return run_decode(prm, head_dim, scale, dtype, num_partitions, (cudaStream_t)stream);
}


namespace pa {
namespace {
// A side stream per device on which pa_decode_shared_prefix runs the shared
// prompt's pass concurrently with the suffix pass on the caller's stream
// (fork and join by events, which stream capture also records). Created on
// first use with that device current, and again after a device reset.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  uint64_t ctx = 0;
};
SideStream g_side[64];
std::mutex g_side_mu;  // held from the fork to the join, so concurrent callers never share an event record

int side_stream_locked(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e, "shared prefix: current device");
  if (dev < 0 || dev >= 64) return PA_ERR_UNSUPPORTED;
  SideStream& ss = g_side[dev];
  const uint64_t now = current_context_id();
  if (ss.stream == nullptr || now == 0 || now != ss.ctx) {
    SideStream fresh;
    e = cudaStreamCreateWithFlags(&fresh.stream, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fresh.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fresh.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return record_cuda_error(e, "shared prefix: create the side stream");
    fresh.ctx = current_context_id();
    ss = fresh;  // handles of a context that a reset destroyed are gone with it
  }
  *out = &ss;
  return PA_OK;
}
}  // namespace
}  // namespace pa

extern "C" PA_API int pa_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                                              void* k_cache, void* v_cache, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                              int num_blocks, int prefix_len, int group_size, float* part_o,
                                              float* part_m, float* part_l, int num_partitions, float scale,
                                              pa_dtype dtype, void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (!out || !part_o || !part_m || !part_l) return PA_ERR_NULL;
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_NULL;
  if ((k_new && !aligned16(k_new)) || (v_new && !aligned16(v_new)) || !aligned16(part_o)) return PA_ERR_ALIGN;
  if (prefix_len <= 0 || prefix_len % kTile || prefix_len % block_size || group_size < 0 || group_size > num_seqs)
    return PA_ERR_SHAPE;
  if (num_partitions < 2) return PA_ERR_WORKSPACE;
  if (num_seqs > 65535) return PA_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  // The prefix pass runs beside the suffix pass, one CTA per SM, so it should
  // hold few SMs: its keys are cut into more than one range (up to 4, each a
  // multiple of 128 keys) only when a range would exceed 4096 keys. Its slots
  // are 0..splits-1; the suffix pass writes slot `splits`.
  int splits = 1;
  for (int c : {2, 4})
    if (prefix_len / splits > 4096 && prefix_len % (128 * c) == 0 && c + 1 <= num_partitions) splits = c;
  // 1) the shared prefix, once for the whole group, on the tensor cores. It
  //    reads no row that pass 2 writes (the appended rows lie past the prefix)
  //    and writes other partial slots, so it runs on a side stream while pass
  //    2 runs on the caller's stream; the merge waits for both.
  std::unique_lock<std::mutex> side_lock(g_side_mu, std::defer_lock);
  SideStream* side = nullptr;
  int prefix_st = PA_OK;
  if (group_size > 0) {
    side_lock.lock();
    st = side_stream_locked(&side);
    if (st != PA_OK) return st;
    cudaError_t e = cudaEventRecord(side->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
    if (e != cudaSuccess) return record_cuda_error(e, "shared prefix: fork to the side stream");
    PrefixPartials pp{prefix_len, part_o, part_m, part_l, num_partitions, splits};
    prefix_st = prefill_tcgen05(nullptr, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, 1,
                                group_size, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype,
                                side->stream, &pp);
    e = cudaEventRecord(side->join, side->stream);
    if (e != cudaSuccess) return record_cuda_error(e, "shared prefix: record the join");
  }
  // 2) every sequence's own tokens in one pass per (sequence, KV head): group
  //    members from prefix_len on (partials), the others whole (final rows);
  //    the newest token's K/V written on the way when given
  DecodeParams prm{};
  prm.out = out;
  prm.part_o = part_o;
  prm.part_m = part_m;
  prm.part_l = part_l;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.k_new = k_new;
  prm.v_new = v_new;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.max_blocks = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.block_size = block_size;
  prm.num_blocks = num_blocks;
  prm.partition = 0;
  prm.num_parts = num_partitions;
  prm.cascade_prefix = prefix_len;
  prm.cascade_group = group_size;
  prm.cascade_slot = splits;
  prm.longest_first = num_seqs > 1 && num_seqs <= PA_DECODE_LPT_MAX_SEQS;
  prm.pair_from = decode_pair_from(num_seqs, num_kv_heads);
  st = run_decode(prm, head_dim, scale, dtype, 1, s);
  if (group_size == 0) return st;
  const cudaError_t e = cudaStreamWaitEvent(s, side->join, 0);  // join, whatever happened above
  side_lock.unlock();
  if (e != cudaSuccess) return record_cuda_error(e, "shared prefix: join the side stream");
  if (prefix_st != PA_OK) return prefix_st;
  if (st != PA_OK) return st;
  // 3) the group's rows: log-sum-exp merge of the prefix slots and the suffix slot
  return launch_merge_any(out, part_o, part_m, part_l, context_lens, group_size * num_q_heads, num_q_heads,
                          head_dim, -(splits + 1), num_partitions, dtype, s);
}

// ---------------------------------------------------------------------------
// pa_decode_splitkv_noalloc: split-KV decode plus merge without any device
// allocation by the caller or by the library.
//
// Some callers cannot hand this library a workspace: a plugin or FFI host
// that exposes no device allocator, a serving runtime that has already given
// all free HBM to its KV block pool, or a latency-critical loop where
// cudaMalloc's implicit device synchronisation is not acceptable. For them
// the partials of the split-KV pass live in a fixed array in the library's
// own device memory (kNoAllocScratchBytes per GPU that loads the library,
// held until the process exits). The caller still passes q, the caches, the
// tables and the output.
// ---------------------------------------------------------------------------
namespace pa {
namespace noalloc {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
static ContextCached<unsigned char*> g_scratch_dev[kMaxDevices];
static std::mutex g_scratch_mu;

// Device address of g_scratch on the current device. In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached together with the identity of
// the context it was taken in: after a device reset the array lives at a new
// address, and the next call looks it up again.
static int scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_dev[dev].valid()) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return record_cuda_error(e, "noalloc: look up the scratch array's device address");
    if (p == nullptr) return PA_ERR_CUDA;
    g_scratch_dev[dev].set(static_cast<unsigned char*>(p));
  }
  *out = g_scratch_dev[dev].value;
  return PA_OK;
}

}  // namespace noalloc
}  // namespace pa

extern "C" PA_API size_t pa_noalloc_scratch_bytes(void) { return pa::noalloc::kNoAllocScratchBytes; }

extern "C" PA_API int pa_decode_splitkv_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                                const int32_t* block_tables, int max_blocks_per_seq,
                                                const int32_t* context_lens, int num_seqs, int num_q_heads,
                                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                int partition_size, int num_partitions, float scale,
                                                pa_dtype dtype, void* stream) {
  int st = check_decode_args(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, dtype);
  if (st != PA_OK || num_seqs == 0) return st;
  if (!out) return PA_ERR_NULL;
  if (partition_size <= 0 || partition_size % kTile || num_partitions <= 0) return PA_ERR_WORKSPACE;
  if (num_seqs > 65535 || num_partitions > (1 << 30)) return PA_ERR_SHAPE;
  // Partials: o [rows, NP, D], then m and l [rows, NP], each start 256-byte
  // aligned. The partition count is compared by division first, so that no
  // product below can wrap around for any accepted shape.
  const size_t rows = static_cast<size_t>(num_seqs) * static_cast<size_t>(num_q_heads);
  const size_t cell_bytes = static_cast<size_t>(head_dim + 2) * sizeof(float);
  if (static_cast<size_t>(num_partitions) > pa::noalloc::kNoAllocScratchBytes / (rows * cell_bytes))
    return PA_ERR_WORKSPACE;
  SplitkvLayout lay;
  if (!splitkv_layout(rows, static_cast<size_t>(num_partitions), static_cast<size_t>(head_dim), &lay) ||
      lay.total > pa::noalloc::kNoAllocScratchBytes)
    return PA_ERR_WORKSPACE;
  unsigned char* base = nullptr;
  st = pa::noalloc::scratch_address(&base);
  if (st != PA_OK) return st;
  float* part_o = reinterpret_cast<float*>(base);
  float* part_m = reinterpret_cast<float*>(base + lay.o_bytes);
  float* part_l = reinterpret_cast<float*>(base + lay.o_bytes + lay.ml_bytes);
  // Every partition p < num_partitions of every row is written by the split
  // pass (empty ones as m = -inf, l = 0, o = 0) before the merge reads it, so
  // nothing left in the array by an earlier call is ever read.
  st = pa_decode_splitkv(part_o, part_m, part_l, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                         context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                         partition_size, num_partitions, scale, dtype, stream);
  if (st != PA_OK) return st;
  return pa_merge(out, part_o, part_m, part_l, context_lens, num_seqs, num_q_heads, head_dim, partition_size,
                  num_partitions, dtype, stream);
}
