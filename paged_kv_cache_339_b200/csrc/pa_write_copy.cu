// pa_write_kv and pa_copy_blocks kernels: bit-exact 16-byte vector copies.
//
// write: each new token's K/V row of one KV head (head_dim elements) goes to
//   pool[slot / BS][head][slot % BS][:]   (slot < 0: padding, skipped)
// at the positions the in-block storage order gives (pa_common.cuh).
// "Paged Attention: Virtual Memory for the KV Cache", "The fix borrowed from
// operating systems": a request fills its current block, then asks for more.
//
// copy: block dst of both pools becomes a copy of block src, all heads: the
// copy a diverging sequence gets of a shared block ("Sharing comes almost for
// free").
//
// swap: the same block copy between the device pools and a host pool the
// device can address (preemption by swapping, "What it does not fix"); the
// kernel reads or writes host memory directly over the host link.
//
// Both are grid-stride loops over 16-byte vectors so consecutive threads touch
// consecutive bytes of a row (coalesced on both sides). Indices outside the
// pool are skipped, never dereferenced.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads)
    write_kv_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                    const uint4* __restrict__ key,
                    const uint4* __restrict__ value,
                    const int64_t* __restrict__ slots, int32_t num_tokens,
                    int32_t num_kv_heads, int32_t block_size,
                    int32_t row_vecs, int32_t head_dim, int64_t num_slots) {
  pdl_launch_dependents();   // the decode plan may start; it waits for us before it ends
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * row_vecs;
  const int64_t total = per_token * num_tokens;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       idx < total; idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / per_token;
    const int64_t r = idx - t * per_token;  // = head * row_vecs + vec
    const int64_t slot = slots[t];
    if (slot < 0 || slot >= num_slots) continue;
    const int64_t blk = slot / block_size;
    const int64_t off = slot - blk * block_size;
    const int64_t h = r / row_vecs;
    const int64_t v = r - h * row_vecs;
    // a 16-byte vector never straddles a 64-element half of the row
    const int vec_elems = head_dim / row_vecs;
    const int64_t in_tile =
        tile_offset(static_cast<int>(off), static_cast<int>(v) * vec_elems, block_size, head_dim) /
        vec_elems;
    const int64_t dst = (blk * num_kv_heads + h) * block_size * row_vecs + in_tile;
    kc[dst] = key[idx];
    vc[dst] = value[idx];
  }
}

__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                       const int64_t* __restrict__ pairs, int32_t num_pairs,
                       int64_t block_vecs, int32_t num_blocks) {
  pdl_launch_dependents();
  const int64_t total = block_vecs * num_pairs;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       idx < total; idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = idx / block_vecs;
    const int64_t v = idx - p * block_vecs;
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) continue;
    kc[dst * block_vecs + v] = kc[src * block_vecs + v];
    vc[dst * block_vecs + v] = vc[src * block_vecs + v];
  }
}

__global__ void __launch_bounds__(kCopyThreads)
    swap_blocks_kernel(uint4* __restrict__ dk, uint4* __restrict__ dv,
                       const uint4* __restrict__ sk, const uint4* __restrict__ sv,
                       const int64_t* __restrict__ pairs, int32_t num_pairs, int64_t block_vecs,
                       int32_t src_blocks, int32_t dst_blocks) {
  const int64_t total = block_vecs * num_pairs;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       idx < total; idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = idx / block_vecs;
    const int64_t v = idx - p * block_vecs;
    const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) continue;
    dk[dst * block_vecs + v] = sk[src * block_vecs + v];
    dv[dst * block_vecs + v] = sv[src * block_vecs + v];
  }
}

int grid_for(int64_t work) {
  const int64_t want = (work + kCopyThreads - 1) / kCopyThreads;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace

cudaError_t launch_write_kv(void* k_cache, void* v_cache, const void* key,
                            const void* value, const int64_t* slots,
                            int32_t num_tokens, int32_t num_kv_heads,
                            int32_t block_size, int32_t row_bytes, int32_t elem_bytes,
                            int64_t num_slots, cudaStream_t stream) {
  const int32_t row_vecs = row_bytes / 16;
  const int64_t work = static_cast<int64_t>(num_tokens) * num_kv_heads * row_vecs;
  write_kv_kernel<<<grid_for(work), kCopyThreads, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), slots,
      num_tokens, num_kv_heads, block_size, row_vecs, row_vecs * 16 / elem_bytes, num_slots);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache,
                               const int64_t* pairs, int32_t num_pairs,
                               int64_t block_bytes, int32_t num_blocks,
                               cudaStream_t stream) {
  const int64_t block_vecs = block_bytes / 16;
  copy_blocks_kernel<<<grid_for(block_vecs * num_pairs), kCopyThreads, 0,
                       stream>>>(static_cast<uint4*>(k_cache),
                                 static_cast<uint4*>(v_cache), pairs,
                                 num_pairs, block_vecs, num_blocks);
  return cudaGetLastError();
}

cudaError_t launch_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* pairs, int32_t num_pairs, int64_t block_bytes,
                               int32_t src_blocks, int32_t dst_blocks, cudaStream_t stream) {
  const int64_t block_vecs = block_bytes / 16;
  swap_blocks_kernel<<<grid_for(block_vecs * num_pairs), kCopyThreads, 0, stream>>>(
      static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), static_cast<const uint4*>(src_k),
      static_cast<const uint4*>(src_v), pairs, num_pairs, block_vecs, src_blocks, dst_blocks);
  return cudaGetLastError();
}

}  // namespace pa
