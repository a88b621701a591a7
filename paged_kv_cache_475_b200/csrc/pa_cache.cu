// Cache-write side of the paged KV cache: slot mapping and the K/V scatter.
//
// [FvP] "Flash Attention vs Paged Attention" 内存管理机制: logical blocks are
// filled left to right; [FP] "FlashAttention y PagedAttention" PagedAttention
// "Cómo funciona" steps 1-3: fixed-size blocks handed out on demand, the block
// table maps logical to physical blocks.
#include "pa_common.cuh"

namespace pa {

__global__ void slot_mapping_kernel(int64_t* __restrict__ slots, const int32_t* __restrict__ block_tables,
                                    int max_blocks, const int32_t* __restrict__ seq_idx,
                                    const int32_t* __restrict__ positions, int num_tokens, int num_seqs,
                                    int block_size, unsigned int* err) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= num_tokens) return;
  const int b = seq_idx[t];
  int64_t slot = -1;
  if (b >= 0) {
    const int pos = positions[t];
    const int j = pos >= 0 ? pos / block_size : -1;
    const int phys = (b < num_seqs && j >= 0 && j < max_blocks)
                         ? block_tables[static_cast<int64_t>(b) * max_blocks + j]
                         : -1;
    if (phys >= 0)
      slot = static_cast<int64_t>(phys) * block_size + pos % block_size;
    else
      set_error(err, PA_DEVERR_POSITION);
  }
  slots[t] = slot;
}

// One thread per 16-byte chunk of a token's [Hkv, D] row, for K and V.
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                         uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                         const int64_t* __restrict__ slots, int num_tokens,
                                         int64_t num_slots, int chunks_per_head, int num_kv_heads,
                                         int block_size, unsigned int* err) {
  const int chunks_per_token = chunks_per_head * num_kv_heads;
  const int64_t total = static_cast<int64_t>(num_tokens) * chunks_per_token;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / chunks_per_token);
    const int c = static_cast<int>(i % chunks_per_token);
    const int64_t s = slots[t];
    if (s < 0) continue;
    if (s >= num_slots) {
      set_error(err, PA_DEVERR_SLOT);
      continue;
    }
    const int h = c / chunks_per_head, cc = c % chunks_per_head;
    const int64_t blk = s / block_size, row = s % block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + row) * chunks_per_head + cc;
    k_cache[dst] = __ldg(k_new + i);
    v_cache[dst] = __ldg(v_new + i);
  }
}

}  // namespace pa

using namespace pa;

extern "C" PA_API int pa_slot_mapping(int64_t* slot_mapping, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* seq_idx,
                                      const int32_t* positions, int num_tokens, int num_seqs,
                                      int block_size, void* stream) {
  if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq < 0) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!slot_mapping || !seq_idx || !positions || (num_seqs > 0 && !block_tables)) return PA_ERR_NULL;
  if (block_size <= 0) return PA_ERR_SHAPE;
  const int threads = 256;
  slot_mapping_kernel<<<(num_tokens + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(
      slot_mapping, block_tables, max_blocks_per_seq, seq_idx, positions, num_tokens, num_seqs, block_size,
      device_error_word());
  return launch_status();
}

extern "C" PA_API int pa_reshape_and_cache(const void* k_new, const void* v_new, void* k_cache,
                                           void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                           int num_blocks, int num_kv_heads, int head_dim, int block_size,
                                           pa_dtype dtype, void* stream) {
  if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_SHAPE;
  if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  const int row_bytes = head_dim * dtype_bytes(dtype);
  if (row_bytes % 16) return PA_ERR_UNSUPPORTED;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_ALIGN;
  const int chunks_per_head = row_bytes / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * chunks_per_head * num_kv_heads;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  reshape_and_cache_kernel<<<blocks, threads, 0, (cudaStream_t)stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_tokens, static_cast<int64_t>(num_blocks) * block_size,
      chunks_per_head, num_kv_heads, block_size, device_error_word());
  return launch_status();
}

// ---------------------------------------------------------------------------
// Whole-block copies between pools: copy-on-write and swap.
//
// [FP] PagedAttention "Cómo funciona" step 4: sequences sharing a prompt
// point at the same physical blocks and copy a block only when their contents
// diverge (copy-on-write); "Flash Attention vs Paged Attention" 恢复机制对比:
// blocks can be swapped out to host memory and back. Both are the same
// operation on a list of (source block, destination block) pairs; the two
// pools may be the same device pool (copy-on-write) or a device pool and a
// pinned host pool (swap out / swap in), which kernels address directly.
// ---------------------------------------------------------------------------
namespace pa {

__global__ void copy_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                   const uint4* __restrict__ src_k, const uint4* __restrict__ src_v,
                                   const int32_t* __restrict__ src_ids, const int32_t* __restrict__ dst_ids,
                                   int num_pairs, int64_t chunks_per_block, int src_blocks, int dst_blocks,
                                   unsigned int* err) {
  const int64_t total = static_cast<int64_t>(num_pairs) * chunks_per_block;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int pr = static_cast<int>(i / chunks_per_block);
    const int64_t c = i % chunks_per_block;
    const int s = src_ids[pr], d = dst_ids[pr];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
      if (c == 0) set_error(err, PA_DEVERR_BLOCK_ID);
      continue;
    }
    dst_k[d * chunks_per_block + c] = src_k[s * chunks_per_block + c];
    dst_v[d * chunks_per_block + c] = src_v[s * chunks_per_block + c];
  }
}

}  // namespace pa

extern "C" PA_API int pa_copy_blocks(void* dst_k, void* dst_v, int dst_num_blocks, const void* src_k,
                                     const void* src_v, int src_num_blocks, const int32_t* src_block_ids,
                                     const int32_t* dst_block_ids, int num_pairs, int num_kv_heads, int head_dim,
                                     int block_size, pa_dtype dtype, void* stream) {
  if (num_pairs < 0 || dst_num_blocks < 0 || src_num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0)
    return PA_ERR_SHAPE;
  if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_pairs == 0) return PA_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !src_block_ids || !dst_block_ids) return PA_ERR_NULL;
  if (!aligned16(dst_k) || !aligned16(dst_v) || !aligned16(src_k) || !aligned16(src_v)) return PA_ERR_ALIGN;
  const int64_t block_bytes = static_cast<int64_t>(num_kv_heads) * block_size * head_dim * dtype_bytes(dtype);
  if (block_bytes % 16) return PA_ERR_UNSUPPORTED;
  const int64_t chunks = block_bytes / 16;
  const int64_t total = chunks * num_pairs;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  copy_blocks_kernel<<<blocks, threads, 0, (cudaStream_t)stream>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), src_block_ids, dst_block_ids, num_pairs, chunks, src_num_blocks,
      dst_num_blocks, device_error_word());
  return launch_status();
}
