/*
 * pa.h - C ABI of the paged-KV attention library (libpa.so, sm_100a / B200).
 *
 * The library computes attention, softmax(q K^T * scale) V, for queries whose
 * keys and values live in a paged KV cache: each sequence's K/V rows sit in
 * fixed-size physical blocks of a shared pool, and a per-sequence block table
 * maps logical block j (tokens j*B .. j*B+B-1) to a physical block id. The
 * softmax is evaluated online (running max and running sum per query row), so
 * no score row is ever written to memory.
 *
 * Sources (web pages, cited by title and section):
 *   [FP]  "FlashAttention y PagedAttention: dos soluciones para dos cuellos de
 *         botella distintos": the attention formula ("Por qué la atención sale
 *         cara"), online softmax and fusion (FlashAttention, "Cómo funciona"),
 *         fixed-size blocks, block tables, sharing and the gather kernel
 *         (PagedAttention, "Cómo funciona", steps 1-5).
 *   [FvP] "Flash Attention vs Paged Attention：大语言模型注意力计算的内存管理革命":
 *         the block-wise formula, eq. (4) (算法原理), left-to-right fill of
 *         logical blocks (内存管理机制), causal-mask fusion and skipping of
 *         masked work (Flash Attention的kernel fusion技术).
 *   [PR]  "Cómo PagedAttention y RadixAttention optimizan el manejo del KV
 *         cache en LLMs": the kernel consults the block table to gather keys
 *         and values ("Cómo funciona PagedAttention", step 2).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument except `stream` and host output pointers is a
 *   device pointer. The caller owns every buffer; the library allocates no
 *   device memory. All tensors are dense, row-major, and 16-byte aligned.
 * - Layouts:
 *     q            [N, Hq, D]      (decode)     [N, C, Hq, D] (prefill chunk)
 *     out          same shape and dtype as q
 *     k_cache      [P, Hkv, B, D]  one (block, kv head) page is B*D contiguous
 *     v_cache      [P, Hkv, B, D]
 *     block_tables int32 [N, max_blocks_per_seq]; entries at or past
 *                  ceil(context_lens[b] / B) are never read (may be -1)
 *     context_lens int32 [N]: keys visible to the sequence's last query,
 *                  including the tokens of the current step
 *   with N sequences, Hq query heads, Hkv KV heads, G = Hq/Hkv, D head dim,
 *   B block size, P pool blocks. Query head h reads KV head h / G.
 * - Supported: D in {64, 128}; B in {8, 16, 32, 64, 128}; G in {1, 2, 4, 8};
 *   dtype f32, f16 or bf16 (prefill: f16 or bf16). Arithmetic is fp32;
 *   outputs are rounded to the input dtype with round-to-nearest-even.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream). Every call is asynchronous on it; the status it returns reports
 *   host-side argument checks and launch errors only.
 * - Device-side checks never trap: a block id outside [0, P), a context
 *   length beyond the block table, a slot outside the pool or a copy that
 *   does not arrive within its wait limit sets a bit in the device error word
 *   (pa_read_error_flags) and the offending access is skipped.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define PA_API __declspec(dllexport)
#else
#define PA_API __attribute__((visibility("default")))
#endif

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_NULL = -1,        /* a required pointer is NULL */
  PA_ERR_SHAPE = -2,       /* a size is negative, zero where it must not be, or inconsistent */
  PA_ERR_DTYPE = -3,       /* unknown dtype, or one the entry point does not take */
  PA_ERR_UNSUPPORTED = -4, /* head dim, block size or group size outside the supported set */
  PA_ERR_WORKSPACE = -5,   /* split-KV partition size / count cannot hold the context */
  PA_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
  PA_ERR_ALIGN = -7        /* a pointer is not 16-byte aligned */
} pa_status;

/* Device error word bits (pa_read_error_flags). */
#define PA_DEVERR_BLOCK_ID 0x1u    /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT 0x2u     /* context length < 0 or beyond max_blocks_per_seq * B */
#define PA_DEVERR_SLOT 0x4u        /* slot_mapping entry outside the pool */
#define PA_DEVERR_WAIT 0x8u        /* an asynchronous copy did not land within its wait limit */
#define PA_DEVERR_POSITION 0x10u   /* slot mapping: sequence index or position outside the table */
#define PA_DEVERR_SETUP 0x20u      /* a CTA could not set itself up (its shared-memory base not at the
                                      alignment its tensor copies need) and computed nothing */

/*
 * pa_slot_mapping - flat cache slot of each new token.
 *
 * [FvP] 内存管理机制: new tokens fill a sequence's logical blocks left to
 * right, so position pos sits in logical block pos / B at offset pos % B;
 * [FP] step 2 / [PR] step 2: the block table gives the physical block.
 *   slot_mapping[t] = block_tables[seq_idx[t]][positions[t] / B] * B + positions[t] % B
 * seq_idx[t] < 0 marks padding and yields -1. A sequence index >= num_seqs,
 * a negative position, a position past the table or a negative table entry
 * also yields -1 and sets PA_DEVERR_POSITION.
 *   slot_mapping  out, int64 [num_tokens]
 *   block_tables  int32 [num_seqs, max_blocks_per_seq]
 *   seq_idx       int32 [num_tokens]   positions int32 [num_tokens]
 * num_tokens == 0 is a no-op.
 */
PA_API int pa_slot_mapping(int64_t* slot_mapping, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* seq_idx,
                           const int32_t* positions, int num_tokens, int num_seqs,
                           int block_size, void* stream);

/*
 * pa_reshape_and_cache - write new K/V rows into their cache slots.
 *
 * [FP] PagedAttention "Cómo funciona" steps 1-3 (blocks filled on demand):
 *   k_cache[s / B, h, s % B, :] = k_new[t, h, :]  for every KV head h,
 *   with s = slot_mapping[t]; the same for V. Bits are copied unchanged.
 * slot < 0 is padding and writes nothing; slot >= num_blocks * B writes
 * nothing and sets PA_DEVERR_SLOT. Two tokens with the same slot in one call
 * give an undefined row. k_new/v_new: [num_tokens, Hkv, D] in `dtype`.
 * num_tokens == 0 is a no-op.
 */
PA_API int pa_reshape_and_cache(const void* k_new, const void* v_new, void* k_cache,
                                void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                int num_blocks, int num_kv_heads, int head_dim,
                                int block_size, pa_dtype dtype, void* stream);

/*
 * pa_copy_blocks - copy whole blocks (all KV heads, K and V) between pools.
 *
 * For each i < num_pairs: dst[dst_block_ids[i]] = src[src_block_ids[i]] in
 * both the K and the V pool, bits unchanged. Covers the copy-on-write of
 * [FP] PagedAttention "Cómo funciona" step 4 (dst pool == src pool: a
 * sequence that diverges inside a shared block gets its own copy) and the
 * swapping of "Flash Attention vs Paged Attention" 恢复机制对比 (one pool in
 * pinned host memory, which kernels address directly: swap out = device to
 * host, swap in = host to device). Pools are [num_blocks, Hkv, B, D] in
 * `dtype`; the id arrays (int32 [num_pairs]) must be device-accessible.
 * An id outside its pool skips that pair and sets PA_DEVERR_BLOCK_ID. A
 * destination that is also a source in the same call gives undefined rows.
 */
PA_API int pa_copy_blocks(void* dst_k, void* dst_v, int dst_num_blocks, const void* src_k,
                          const void* src_v, int src_num_blocks, const int32_t* src_block_ids,
                          const int32_t* dst_block_ids, int num_pairs, int num_kv_heads,
                          int head_dim, int block_size, pa_dtype dtype, void* stream);

/*
 * pa_decode - one query token per sequence over its whole paged context.
 *
 * out[b, h, :] = sum_t softmax_t(scale * q[b,h,:] . K_b[t]) V_b[t], t < context_lens[b],
 * with K_b/V_b read through block_tables[b] ([FP] "Por qué la atención sale
 * cara" for the formula; [FP] PagedAttention step 5 and [PR] step 2 for the
 * gather). One pass: each K/V page is read once for all G query heads of its
 * group, and the softmax is kept online ([FP] FlashAttention "Cómo funciona").
 * context_lens[b] == 0 gives a zero row.
 */
PA_API int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int max_blocks_per_seq,
                     const int32_t* context_lens, int num_seqs, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     float scale, pa_dtype dtype, void* stream);

/*
 * pa_decode_append - pa_decode with the step's cache write folded in.
 *
 * For decode steps that append exactly one token per sequence, at position
 * context_lens[b] - 1: first the token's rows are written into its slot,
 *   k_cache[phys, h, (L_b-1) % B, :] = k_new[b, h, :]   (same for V, every KV head h,
 *   phys = block_tables[b][(L_b-1) / B]),
 * exactly as pa_slot_mapping + pa_reshape_and_cache would ([FvP] 内存管理机制,
 * [FP] PagedAttention steps 1-3), then the output is pa_decode's. One launch
 * instead of three: the CTA that reads the newest token's page writes the
 * row itself before its bulk copies read it. k_new/v_new: [N, Hkv, D].
 * A bad block id for the newest position skips the write and sets
 * PA_DEVERR_BLOCK_ID. Its page must not be shared with another sequence.
 */
PA_API int pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float scale, pa_dtype dtype, void* stream);

/* Number of partitions of `partition_size` tokens a context of
 * max_context_len tokens needs (at least 1; 0 if partition_size <= 0). */
PA_API int pa_splitkv_num_partitions(int max_context_len, int partition_size);

/*
 * pa_splitkv_workspace_bytes - size of one caller-owned buffer that holds all
 * three split-KV partial arrays of pa_decode_splitkv / pa_merge for N
 * sequences, Hq query heads, head dim D, contexts of at most max_context_len
 * tokens and partitions of partition_size tokens. With
 * NP = pa_splitkv_num_partitions(max_context_len, partition_size) and every
 * part rounded up to a multiple of 256 bytes, the buffer holds
 *   part_o float [N, Hq, NP, D] at byte 0,
 *   part_m float [N, Hq, NP]    at byte round256(N*Hq*NP*D*4),
 *   part_l float [N, Hq, NP]    right after part_m, at round256(...) + round256(N*Hq*NP*4).
 * (The split partials are the per-block sums of [FvP] eq. (4); the pages fix
 * no memory layout for them.) Pure host arithmetic, no CUDA call. Returns 0
 * when N == 0, when an argument is negative (N, max_context_len) or not
 * positive (Hq, D, partition_size), or when the size does not fit in size_t.
 */
PA_API size_t pa_splitkv_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                         int partition_size);

/*
 * pa_decode_splitkv - per-partition online-softmax state of a decode step.
 *
 * Partition p of sequence b covers tokens [p*S, min((p+1)*S, L_b)), S =
 * partition_size (a positive multiple of 16). For every (b, h, p):
 *   part_m[b,h,p] = max_t s_t              (s_t = scale * q[b,h,:] . K_b[t], natural-log units)
 *   part_l[b,h,p] = sum_t exp(s_t - part_m)
 *   part_o[b,h,p,:] = sum_t exp(s_t - part_m) V_b[t]   (unnormalised, fp32)
 * This is the running max / running sum of [FP] FlashAttention "Cómo
 * funciona", and the per-block sums of [FvP] eq. (4), taken one partition at
 * a time. Partitions at or past ceil(L_b / S) (and every partition of an
 * empty context) are written as m = -inf, l = 0, o = 0.
 *   part_o [N, Hq, num_partitions, D]  part_m, part_l [N, Hq, num_partitions]  (fp32)
 * num_partitions must be >= ceil(max_b L_b / S), else the tail is dropped and
 * PA_DEVERR_CONTEXT is set; pa_splitkv_num_partitions gives the count.
 */
PA_API int pa_decode_splitkv(float* part_o, float* part_m, float* part_l, const void* q,
                             const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                             int partition_size, int num_partitions, float scale,
                             pa_dtype dtype, void* stream);

/*
 * pa_decode_shared_prefix - decode for a batch whose first `group_size`
 * sequences share their first `prefix_len` tokens through the same physical
 * blocks (a common prompt: [FP] PagedAttention step 4 and its block-table
 * example; [PR], RadixAttention's reuse of a prefix's KV state).
 *
 * Same output as pa_decode (plus, when k_new/v_new are given, the cache write
 * of pa_decode_append), computed as a cascade:
 *   1) the group's G*group_size query rows of each KV head attend to the shared
 *      prefix pages once, as a dense tile on the tensor cores (read through
 *      block_tables row 0); the prefix keys form S equal ranges, one partial
 *      slot each: S = 1, or 2 or 4 when a range would otherwise exceed 4096
 *      keys (ranges are multiples of 128 keys, S + 1 <= num_partitions);
 *   2) one pass per (sequence, KV head) over the sequence's own tokens: group
 *      members from token prefix_len on, written as partials into slot S; all
 *      other sequences whole, written straight to `out`; the newest token's
 *      row written first if given;
 *   3) the group's rows: log-sum-exp merge of slots 0..S.
 * Passes 1 and 2 touch disjoint data, so pass 1 runs on a stream the library
 * keeps per device (created on the first call with that device current, and
 * again after a device reset), forked from and joined back to `stream` by
 * events before pass 3; stream capture records the fork and the join.
 * part_o/part_m/part_l: caller workspace [N, Hq, num_partitions(, D)] fp32,
 * num_partitions >= 2 (5 lets S reach 4). Needs prefix_len a positive
 * multiple of 16 and of B, every group member with L_b > prefix_len (else
 * PA_DEVERR_CONTEXT), f16 or bf16. The kernels do not check that the prefix
 * blocks are really shared.
 */
PA_API int pa_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                                   void* k_cache, void* v_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                   int num_blocks, int prefix_len, int group_size, float* part_o,
                                   float* part_m, float* part_l, int num_partitions, float scale,
                                   pa_dtype dtype, void* stream);

/*
 * pa_decode_splitkv_append - pa_decode_splitkv with the step's cache write
 * folded in, like pa_decode_append: the CTA whose partition holds position
 * context_lens[b] - 1 writes k_new[b] / v_new[b] ([N, Hkv, D]) into that slot
 * before reading it. Same partials and requirements as pa_decode_splitkv.
 */
PA_API int pa_decode_splitkv_append(float* part_o, float* part_m, float* part_l, const void* q,
                                    const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                                    const int32_t* block_tables, int max_blocks_per_seq,
                                    const int32_t* context_lens, int num_seqs, int num_q_heads,
                                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                    int partition_size, int num_partitions, float scale, pa_dtype dtype,
                                    void* stream);

/*
 * pa_merge - combine split-KV partitions into the attention output.
 *
 * Log-sum-exp rule over the partitions p < ceil(L_b / S) with part_l > 0
 * (the online-softmax update of [FP] applied across partitions):
 *   M = max_p m_p,  Lsum = sum_p exp(m_p - M) l_p,
 *   out[b,h,:] = sum_p exp(m_p - M) o_p / Lsum   (rounded to `dtype`)
 * A row with no such partition is zero. context_lens and partition_size
 * must be the ones given to pa_decode_splitkv: with them the merge reads only
 * the ceil(L_b / S) partitions that hold tokens of row b and never touches
 * the slots of partitions past a short row's context (the pages give no
 * merge interface; this is the reading of the log-sum-exp rule used here).
 */
PA_API int pa_merge(void* out, const float* part_o, const float* part_m, const float* part_l,
                    const int32_t* context_lens, int num_seqs, int num_q_heads, int head_dim,
                    int partition_size, int num_partitions, pa_dtype dtype, void* stream);

/*
 * pa_prefill_chunk - C causal query tokens per sequence over its paged context.
 *
 * Query i of sequence b sits at position p = L_b - C + i (context_lens
 * counts the chunk, whose K/V rows pa_reshape_and_cache has already written)
 * and attends to keys 0..p: the whole earlier context plus the chunk's keys up
 * to itself ([FvP] eq. (4): the block sum stops at the block holding the
 * query, cut at the query's own token). Key tiles wholly past a query tile's
 * last position are not computed ([FvP] kernel fusion: skipping masked work).
 * Rows with p < 0 (L_b < C) are zero. q/out: [N, C, Hq, D]; f16 or bf16.
 */
PA_API int pa_prefill_chunk(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int num_seqs, int chunk_len,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float scale, pa_dtype dtype, void* stream);

/*
 * pa_decode_splitkv_noalloc - split-KV decode and merge in one call, with no
 * device memory allocated by the caller or by the library. (The pages have
 * no counterpart of this entry point; it exists for callers that cannot
 * allocate.)
 *
 * Same result as pa_decode_splitkv followed by pa_merge, written to `out`
 * [N, Hq, D]. It is meant for callers that cannot provide a workspace: a
 * plugin or FFI host with no device allocator at hand, a serving runtime
 * that has already handed all free HBM to its KV block pool, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device
 * synchronisation. The partials live instead in a fixed array inside the
 * library's own device memory, pa_noalloc_scratch_bytes() = 16 MiB on every
 * GPU that loads the library, held until the process exits. The call needs
 * N * Hq * num_partitions * (D + 2) * 4 bytes of it (each part rounded up to
 * 256 bytes); larger requests return PA_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture begins. The address is remembered together with the CUDA context
 * it was taken in: after cudaDeviceReset the array lives at a new address,
 * and the next call on that device looks it up again (so make that call
 * outside a stream capture too). Every call on a device shares the one
 * array: calls whose kernels overlap on the GPU (other streams, other host
 * threads) race and must be serialised by the caller. Nothing in the array
 * needs clearing: each call writes every partial it later reads.
 * N * Hq * num_partitions is checked against the array size before any
 * product is formed, so no accepted shape can wrap the size arithmetic;
 * num_partitions > 2^30 returns PA_ERR_SHAPE.
 */
PA_API int pa_decode_splitkv_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int max_blocks_per_seq,
                                     const int32_t* context_lens, int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                     int partition_size, int num_partitions, float scale,
                                     pa_dtype dtype, void* stream);

/*
 * pa_decode_selftest_starved_wait - self-test of the copy-wait time-out; not
 * part of the attention path. Runs pa_decode (same arguments, same checks)
 * except that warp 0 of the first CTA arms its first copy stage for a tile
 * whose copies are never issued, and every copy wait gives up after
 * wait_cycles SM cycles (1000 .. 4e9; else PA_ERR_SHAPE). That wait runs out:
 * the warp sets PA_DEVERR_WAIT, waits (same limit) for its copies that were
 * issued, and the CTA finishes; rows of that CTA (KV head 0 of the longest
 * sequence, the lowest index among equals; of sequence 0 when num_seqs is 1
 * or above 512) are then undefined, all other rows are those of pa_decode. Nothing
 * stays in flight, so the context remains usable. f16 with head_dim 128 only
 * (else PA_ERR_UNSUPPORTED). Returns the launch status.
 */
PA_API int pa_decode_selftest_starved_wait(void* out, const void* q, const void* k_cache, const void* v_cache,
                                           const int32_t* block_tables, int max_blocks_per_seq,
                                           const int32_t* context_lens, int num_seqs, int num_q_heads,
                                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                           float scale, pa_dtype dtype, long long wait_cycles, void* stream);

/* Size in bytes of the per-device array pa_decode_splitkv_noalloc works in. */
PA_API size_t pa_noalloc_scratch_bytes(void);

/*
 * pa_read_error_flags - read (and optionally clear) the device error word of
 * the current device. Synchronises the device. Returns PA_OK or PA_ERR_CUDA.
 */
PA_API int pa_read_error_flags(uint32_t* host_flags, int clear);

/* Message of the last CUDA failure behind a PA_ERR_CUDA returned on this host
 * thread (the failing step, CUDA's error string and name); "" if none. */
PA_API const char* pa_last_cuda_error(void);

/* Human-readable name of a pa_status value. */
PA_API const char* pa_status_string(int status);

/*
 * Timeline tracing, for builds made with -DPA_TRACE=1 (python
 * paged_kv_cache_475_b200/build.py --trace); every other build returns
 * PA_ERR_UNSUPPORTED from both calls. A traced decode kernel writes one
 * record per CTA (linear CTA index, at most 65536) into a device array:
 *   struct { uint64 t_start, t_first, t_end;   global timer, ns: entry, first
 *                                               tile landed (warp 0), exit
 *            int32 smid, seq, kv_head, part, tokens, kind; }  (48 bytes)
 * pa_trace_clear zeroes the array (synchronises); pa_trace_read synchronises
 * and copies max_records records to host memory. The records of the last
 * traced launch overwrite those of earlier ones. Not part of the attention
 * path: the pages have no counterpart; it measures where a kernel's time goes.
 */
PA_API int pa_trace_clear(void);
PA_API int pa_trace_read(void* host_records, int max_records);

/* Library ABI version (major * 100 + minor): 101 adds pa_splitkv_workspace_bytes,
 * 102 pa_decode_selftest_starved_wait. */
PA_API int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
